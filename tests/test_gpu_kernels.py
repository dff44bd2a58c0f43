"""GPU parity of each kernel against the fp64 oracle on seeded inputs, called
through the C ABI.  Sizes span several tiles with ragged tails."""
import math

import numpy as np
import pytest

from oracle import dit_oracle as O
from diffusion_transformer_block_flux_b200 import synth
import diffusion_transformer_block_flux_b200 as dit
from helpers import dev_bf16, dev_tree, host_f64, parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    dit.lib()
    yield
    torch.cuda.synchronize()


def f32dev(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def assert_no_device_error():
    st, code = dit.dit_get_device_error()
    assert st == 0 and code == 0, f"device error word {code:#x}"


# ---------------------------------------------------------------- RoPE table

@pytest.mark.parametrize("pairs,axes,ids_fn", [
    ((8, 28, 28), (16, 56, 56), lambda: synth.flux_ids(64, 12, 16)),
    ((22, 21, 21), (44, 42, 42), lambda: synth.video_ids(3, 5, 7)),
])
def test_rope_table(pairs, axes, ids_fn):
    import torch
    ids = ids_fn()
    S = ids.shape[0]
    rope = torch.empty((S, 64, 2), dtype=torch.float32, device="cuda")
    dit.dit_rope_table(torch.from_numpy(ids).cuda(), pairs, 10000.0, rope)
    phi = O.rope_angles(ids, axes)
    got = rope.cpu().double().numpy()
    assert np.abs(got[..., 0] - np.cos(phi)).max() < 1e-6
    assert np.abs(got[..., 1] - np.sin(phi)).max() < 1e-6


# ---------------------------------------------------------------- adaLN

@pytest.mark.parametrize("B,N,K", [(1, 1152, 384), (2, 9216, 3072), (3, 200, 64), (1, 9216, 3072), (1, 18432, 3072),
                                   (1, 1001, 4096), (1, 37, 256), (1, 5, 1536)])
def test_adaln_modulation(B, N, K):
    import torch
    vec = synth.normal_bf16(1, "vec", (B, K))
    W = synth.normal_bf16(0, "W", (N, K), 0.02)
    b = synth.normal_bf16(0, "b", (N,), 0.1)
    out = torch.empty((B, N), dtype=torch.float32, device="cuda")
    dit.dit_adaln_modulation(dev_bf16(vec), dev_bf16(W), dev_bf16(b), out)
    ref = O.linear(O.silu(synth.bf16_bits_to_f64(vec)), synth.bf16_bits_to_f64(W), synth.bf16_bits_to_f64(b))
    rl2, _ = parity(out.cpu().double().numpy(), ref, "adaln")
    assert rl2 < 1e-4  # fp32 output, fp32 accumulation


def test_vec_linear_bf16_out_no_silu():
    import torch
    x = synth.normal_bf16(1, "x", (1, 256))
    W = synth.normal_bf16(0, "W", (384, 256), 0.02)
    out = torch.empty((1, 384), dtype=torch.bfloat16, device="cuda")
    dit.dit_vec_linear(dev_bf16(x), dev_bf16(W), None, out, flags=dit.DIT_VEC_OUT_BF16)
    ref = O.linear(synth.bf16_bits_to_f64(x), synth.bf16_bits_to_f64(W))
    parity(host_f64(out), ref, "vec_linear")


# ---------------------------------------------------------------- LayerNorm + modulate

@pytest.mark.parametrize("B,S,D", [(2, 100, 384), (1, 37, 3072), (1, 5, 1536), (1, 3, 8), (1, 4608, 3072),
                                   (2, 1301, 1536), (1, 333, 8192), (3, 257, 512), (1, 1000, 6144)])
def test_modulate_norm(B, S, D):
    import torch
    x = synth.normal_bf16(1, "x", (B * S, D), 2.0, 0.5)
    sh = synth.bf16_bits_to_f64(synth.normal_bf16(2, "sh", (B, D), 0.7))
    sc = synth.bf16_bits_to_f64(synth.normal_bf16(3, "sc", (B, D), 0.7))
    y = torch.empty((B * S, D), dtype=torch.bfloat16, device="cuda")
    dit.dit_modulate_norm(dev_bf16(x), f32dev(sh), f32dev(sc), y, B, S, mod_stride=D)
    xf = synth.bf16_bits_to_f64(x).reshape(B, S, D)
    ref = O.modulate(O.layer_norm(xf), sh[:, None, :], sc[:, None, :]).reshape(B * S, D)
    parity(host_f64(y), ref, "modulate_norm")
    # plain LayerNorm (no modulation)
    dit.dit_modulate_norm(dev_bf16(x), None, None, y, B, S)
    parity(host_f64(y), O.layer_norm(xf).reshape(B * S, D), "layer_norm")


def test_modulate_norm_equal_and_offset_rows():
    """Rows of one repeated value normalise to exactly 0 (then the shift);
    rows far from zero mean (offset 200, std 1) keep their deviations: the
    statistics are taken about the mean, not as E[x^2] - E[x]^2.  More rows
    than resident CTAs, so every CTA's ring of rows wraps."""
    import torch
    S, D = 2000, 3072
    x = synth.normal_bf16(5, "x", (S, D))
    vals = [0.0, 1.0, -3.5, 1e-3, 448.0, 65536.0]
    for r, c in enumerate(vals):
        x[r] = synth.const_bf16((D,), c)
    off = synth.normal_bf16(6, "off", (8, D), 1.0, 200.0)
    x[len(vals):len(vals) + 8] = off
    sh = synth.bf16_bits_to_f64(synth.normal_bf16(7, "sh", (1, D), 0.7))
    sc = synth.bf16_bits_to_f64(synth.normal_bf16(8, "sc", (1, D), 0.7))
    y = torch.empty((S, D), dtype=torch.bfloat16, device="cuda")
    xf = synth.bf16_bits_to_f64(x)
    dit.dit_modulate_norm(dev_bf16(x), None, None, y, 1, S)
    got = host_f64(y)
    assert np.all(got[:len(vals)] == 0.0), "equal rows must normalise to exactly 0"
    parity(got, O.layer_norm(xf), "layer_norm equal/offset rows")
    dit.dit_modulate_norm(dev_bf16(x), f32dev(sh), f32dev(sc), y, 1, S, mod_stride=D)
    got = host_f64(y)
    ref = O.modulate(O.layer_norm(xf), sh, sc)
    np.testing.assert_array_equal(got[:len(vals)], host_f64(dev_bf16(synth.f32_to_bf16_bits(
        np.broadcast_to(sh.astype(np.float32), (len(vals), D))))))
    parity(got, ref, "modulate_norm equal/offset rows")
    parity(got[len(vals):len(vals) + 8], ref[len(vals):len(vals) + 8], "modulate_norm offset rows")


# ---------------------------------------------------------------- QK RMSNorm + RoPE

@pytest.mark.parametrize("B,nt,gh,gw,H", [(1, 64, 12, 16, 3), (2, 5, 3, 7, 2)])
def test_qk_norm_rope(B, nt, gh, gw, H):
    import torch
    ids = synth.flux_ids(nt, gh, gw)
    S = ids.shape[0]
    D = H * 128
    qkv = synth.normal_bf16(1, "qkv", (B * S, 3 * D), 1.5)
    qs = synth.normal_bf16(0, "qs", (128,), 0.1, 1.0)
    ks = synth.normal_bf16(0, "ks", (128,), 0.1, 1.0)
    rope = torch.empty((S, 64, 2), dtype=torch.float32, device="cuda")
    dit.dit_rope_table(torch.from_numpy(ids).cuda(), (8, 28, 28), 10000.0, rope)
    d_qkv = dev_bf16(qkv)
    qo = torch.empty((B * S, D), dtype=torch.bfloat16, device="cuda")
    ko = torch.empty_like(qo)
    dit.dit_qk_norm_rope(d_qkv[:, :D], d_qkv[:, D:2 * D], dev_bf16(qs), dev_bf16(ks), rope, qo, ko, B, S, H)
    phi = O.rope_angles(ids, (16, 56, 56))
    f = synth.bf16_bits_to_f64(qkv).reshape(B, S, 3 * D)
    for which, out, sc in ((0, qo, qs), (1, ko, ks)):
        ref = np.concatenate([O.apply_rope(O.rms_norm_heads(f[b, :, which * D:(which + 1) * D],
                                                            synth.bf16_bits_to_f64(sc), H), phi, H)
                              for b in range(B)])
        parity(host_f64(out), ref, "qk_norm_rope")
    # in place gives the same bits
    dit.dit_qk_norm_rope(d_qkv[:, :D], d_qkv[:, D:2 * D], dev_bf16(qs), dev_bf16(ks), rope, d_qkv[:, :D],
                         d_qkv[:, D:2 * D], B, S, H)
    assert torch.equal(d_qkv[:, :D], qo) and torch.equal(d_qkv[:, D:2 * D], ko)


# ---------------------------------------------------------------- GEMM + epilogues

def _gemm_inputs(M, N, K, seed=0):
    A = synth.normal_bf16(seed + 1, "A", (M, K))
    W = synth.normal_bf16(seed, "W", (N, K), 0.02)
    b = synth.normal_bf16(seed, "b", (N,), 0.1)
    return A, W, b


@pytest.mark.parametrize("M,N,K", [(300, 2688, 384), (128, 256, 64), (1, 32, 8), (256, 512, 15360),
                                   (777, 96, 200)])
def test_gemm_bias(M, N, K):
    import torch
    A, W, b = _gemm_inputs(M, N, K)
    C = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    dit.dit_gemm_epilogue(dev_bf16(A), dev_bf16(W), C, dit.DIT_EPI_BIAS, bias=dev_bf16(b))
    ref = O.linear(synth.bf16_bits_to_f64(A), synth.bf16_bits_to_f64(W), synth.bf16_bits_to_f64(b))
    parity(host_f64(C), ref, "gemm_bias")
    dit.dit_gemm_epilogue(dev_bf16(A), dev_bf16(W), C, dit.DIT_EPI_NONE)
    parity(host_f64(C), O.linear(synth.bf16_bits_to_f64(A), synth.bf16_bits_to_f64(W)), "gemm_none")
    assert_no_device_error()


def test_gemm_gelu_cols_split_output():
    import torch
    M, D, Mh = 300, 384, 1536
    N, K = 3 * D + Mh, D
    A, W, b = _gemm_inputs(M, N, K, seed=5)
    qkv = torch.empty((M, 3 * D), dtype=torch.bfloat16, device="cuda")
    cat = torch.zeros((M, D + Mh), dtype=torch.bfloat16, device="cuda")
    dit.dit_gemm_epilogue(dev_bf16(A), dev_bf16(W), qkv, dit.DIT_EPI_BIAS_GELU_COLS, bias=dev_bf16(b),
                          C2=cat[:, D:], split_col=3 * D, gelu_col_begin=3 * D)
    h = O.linear(synth.bf16_bits_to_f64(A), synth.bf16_bits_to_f64(W), synth.bf16_bits_to_f64(b))
    parity(host_f64(qkv), h[:, :3 * D], "gemm qkv part")
    parity(host_f64(cat[:, D:]), O.gelu_tanh(h[:, 3 * D:]), "gemm gelu part")
    assert torch.count_nonzero(cat[:, :D]) == 0  # columns left of the split untouched


@pytest.mark.parametrize("norm,B", [(1, 1), (0, 2)])
def test_gemm_fused_qk_norm_rope(norm, B):
    """QKV|MLP GEMM with RMSNorm + RoPE fused into the epilogue for the q and k
    columns (and GELU on the MLP columns, written through the split output)."""
    import torch
    ids = synth.flux_ids(44, 16, 16)  # 300 tokens: ragged last row tile
    S = ids.shape[0]
    H, Mh = 2, 512
    D = H * 128
    N, K = 3 * D + Mh, D
    A, W, b = _gemm_inputs(B * S, N, K, seed=11)
    qs = synth.normal_bf16(0, "qs", (128,), 0.1, 1.0)
    ks = synth.normal_bf16(0, "ks", (128,), 0.1, 1.0)
    rope = torch.empty((S, 64, 2), dtype=torch.float32, device="cuda")
    dit.dit_rope_table(torch.from_numpy(ids).cuda(), (8, 28, 28), 10000.0, rope)
    qkv = torch.empty((B * S, 3 * D), dtype=torch.bfloat16, device="cuda")
    mlp = torch.empty((B * S, Mh), dtype=torch.bfloat16, device="cuda")
    dit.dit_gemm_epilogue(dev_bf16(A), dev_bf16(W), qkv, dit.DIT_EPI_BIAS_GELU_COLS, bias=dev_bf16(b), C2=mlp,
                          split_col=3 * D, gelu_col_begin=3 * D, qk_cols=2 * D, qk_norm=norm,
                          q_scale=dev_bf16(qs), k_scale=dev_bf16(ks), rope=rope, rope_rows=S)
    h = O.linear(synth.bf16_bits_to_f64(A), synth.bf16_bits_to_f64(W), synth.bf16_bits_to_f64(b))
    phi = np.tile(O.rope_angles(ids, (16, 56, 56)), (B, 1))
    got = host_f64(qkv)
    for which, sc in ((0, qs), (1, ks)):
        x = h[:, which * D:(which + 1) * D]
        if norm:
            x = O.rms_norm_heads(x, synth.bf16_bits_to_f64(sc), H)
        else:
            x = x * np.tile(synth.bf16_bits_to_f64(sc), H)
        parity(got[:, which * D:(which + 1) * D], O.apply_rope(x, phi, H), f"fused {'qk'[which]}")
    parity(got[:, 2 * D:], h[:, 2 * D:3 * D], "v columns")
    parity(host_f64(mlp), O.gelu_tanh(h[:, 3 * D:]), "gelu columns")


@pytest.mark.parametrize("M,rows_per_batch,N,K,inplace", [(300, 150, 384, 1920, False), (256, 256, 3072, 512, True)])
def test_gemm_gated_residual(M, rows_per_batch, N, K, inplace):
    import torch
    A, W, b = _gemm_inputs(M, N, K, seed=9)
    B = M // rows_per_batch
    x = synth.normal_bf16(3, "x", (M, N))
    gate = synth.bf16_bits_to_f64(synth.normal_bf16(4, "g", (B, N), 0.7))
    d_x = dev_bf16(x)
    out = d_x if inplace else torch.empty_like(d_x)
    dit.dit_gemm_epilogue(dev_bf16(A), dev_bf16(W), out, dit.DIT_EPI_BIAS_GATED_RESIDUAL, bias=dev_bf16(b),
                          gate=f32dev(gate), gate_stride=N, resid=d_x, rows_per_batch=rows_per_batch)
    y = O.linear(synth.bf16_bits_to_f64(A), synth.bf16_bits_to_f64(W), synth.bf16_bits_to_f64(b))
    xf = synth.bf16_bits_to_f64(x)
    g = np.repeat(gate, rows_per_batch, axis=0)
    ref = xf + g * y
    got = host_f64(out)
    parity(got, ref, "gated residual out")
    # with a small residual the output is the branch itself: same tolerance
    xs = synth.f32_to_bf16_bits(synth.bf16_bits_to_f32(x) * np.float32(2.0 ** -8))
    d_xs = dev_bf16(xs)
    out_s = torch.empty_like(d_xs)
    dit.dit_gemm_epilogue(dev_bf16(A), dev_bf16(W), out_s, dit.DIT_EPI_BIAS_GATED_RESIDUAL, bias=dev_bf16(b),
                          gate=f32dev(gate), gate_stride=N, resid=d_xs, rows_per_batch=rows_per_batch)
    xsf = synth.bf16_bits_to_f64(xs)
    assert np.linalg.norm(g * y) > 10 * np.linalg.norm(xsf)
    parity(host_f64(out_s), xsf + g * y, "gated residual, small residual")


@pytest.mark.parametrize("epi,M1,M2,N1,N2,K", [
    ("gated", 512, 4096, 768, 768, 1536),   # text + image output projections (M1 < N: M-fastest; M2 > N: N-fastest)
    ("gelu", 512, 1000, 1024, 1024, 512),   # MLP-in with GELU, ragged image rows
    ("qk", 300, 700, 768, 768, 256),        # QKV with the fused per-head RMSNorm + RoPE
    ("gelu", 600, 300, 512, 1536, 384),     # jobs of different widths
    ("gated", 100, 600, 256, 256, 512),     # M1 <= 128: two launches
])
def test_gemm_grouped_equals_two_calls(epi, M1, M2, N1, N2, K):
    """Two GEMMs in one grouped launch (the double-stream block's text and
    image layers) give exactly what two dit_gemm_epilogue calls give, and the
    oracle's result within the stated tolerance."""
    import torch
    D = 768
    jobs = []
    for j, (M, N) in enumerate(((M1, N1), (M2, N2))):
        A, W, b = _gemm_inputs(M, N, K, seed=31 + 7 * j)
        t = {"A": dev_bf16(A), "W": dev_bf16(W), "b": dev_bf16(b), "Af": A, "Wf": W, "bf": b, "M": M}
        kw = dict(bias=t["b"])
        if epi == "gated":
            x = synth.normal_bf16(40 + j, "x", (M, N))
            g = synth.bf16_bits_to_f64(synth.normal_bf16(50 + j, "g", (1, N), 0.7))
            t["x"], t["g"] = x, g
            t["resid"] = dev_bf16(x)
            kw.update(epi=dit.DIT_EPI_BIAS_GATED_RESIDUAL, gate=f32dev(g), gate_stride=0, resid=t["resid"])
        elif epi == "gelu":
            kw.update(epi=dit.DIT_EPI_BIAS_GELU_COLS, gelu_col_begin=256)
        else:
            ids = torch.from_numpy(synth.flux_ids(16, 16, (M - 16 + 15) // 16)[:M]).cuda()
            rope = torch.empty((M, 64, 2), dtype=torch.float32, device="cuda")
            dit.dit_rope_table(ids, (8, 28, 28), 10000.0, rope)
            t["rope"] = rope
            kw.update(epi=dit.DIT_EPI_BIAS, qk_cols=2 * (N // 3 // 128) * 128, rope=rope, rope_rows=M)
        t["kw"] = kw
        t["N"] = N
        jobs.append(t)
    sep = [torch.empty((t["M"], t["N"]), dtype=torch.bfloat16, device="cuda") for t in jobs]
    grp = [torch.empty_like(o) for o in sep]
    for t, o in zip(jobs, sep):
        dit.dit_gemm_epilogue(t["A"], t["W"], o, **t["kw"])
    args = [dit.gemm_args(t["A"], t["W"], o, **t["kw"]) for t, o in zip(jobs, grp)]
    dit.dit_gemm_epilogue_grouped(args[0], args[1])
    torch.cuda.synchronize()
    for o_s, o_g in zip(sep, grp):
        assert torch.equal(o_s, o_g)
    if epi != "qk":
        for t, o in zip(jobs, grp):
            y = O.linear(synth.bf16_bits_to_f64(t["Af"]), synth.bf16_bits_to_f64(t["Wf"]),
                         synth.bf16_bits_to_f64(t["bf"]))
            if epi == "gated":
                ref = synth.bf16_bits_to_f64(t["x"]) + t["g"] * y
            else:
                ref = np.concatenate([y[:, :256], O.gelu_tanh(y[:, 256:])], axis=1)
            parity(host_f64(o), ref, f"grouped {epi}, M={t['M']}")
    assert_no_device_error()


def test_weight_l2_persist_changes_no_bits():
    """With the opt-in L2 residency of the output GEMM's weight, the N-fastest
    GEMM (M > N) loads its weight with the evict-last policy and demotes it at
    the end: a caching hint, so the output equals the plain call bit for bit,
    and the oracle's.  The process-wide set-aside is turned off again."""
    import torch
    M, N, K = 1024, 256, 2048
    A, W, b = _gemm_inputs(M, N, K, seed=17)
    x = synth.normal_bf16(5, "x", (M, N))
    gate = synth.bf16_bits_to_f64(synth.normal_bf16(6, "g", (1, N), 0.7))
    dA, dW, db, dx, dg = dev_bf16(A), dev_bf16(W), dev_bf16(b), dev_bf16(x), f32dev(gate)
    plain = torch.empty_like(dx)
    kept = torch.empty_like(dx)
    dit.dit_gemm_epilogue(dA, dW, plain, dit.DIT_EPI_BIAS_GATED_RESIDUAL, bias=db, gate=dg, gate_stride=N, resid=dx)
    try:
        dit.dit_set_weight_l2_persist(64 << 20)
        dit.dit_gemm_epilogue(dA, dW, kept, dit.DIT_EPI_BIAS_GATED_RESIDUAL, bias=db, gate=dg, gate_stride=N,
                              resid=dx)
        torch.cuda.synchronize()
    finally:
        dit.dit_set_weight_l2_persist(0)
    assert torch.equal(plain, kept)
    y = O.linear(synth.bf16_bits_to_f64(A), synth.bf16_bits_to_f64(W), synth.bf16_bits_to_f64(b))
    parity(host_f64(kept), synth.bf16_bits_to_f64(x) + gate * y, "gated residual, weight kept in L2")
    assert_no_device_error()


# ---------------------------------------------------------------- attention

def _attn_case(B, Sq, Skv, H, qmul=1.0, seed=0):
    D = H * 128
    q = synth.normal_bf16(seed + 1, "q", (B * Sq, D), qmul)
    k = synth.normal_bf16(seed + 2, "k", (B * Skv, D))
    v = synth.normal_bf16(seed + 3, "v", (B * Skv, D))
    return q, k, v


@pytest.mark.parametrize("B,Sq,Skv,H,qmul", [
    (1, 256, 256, 3, 1.0),     # tiny single-block shape
    (2, 300, 333, 2, 1.0),     # ragged query and key tails, batch strides
    (1, 384, 640, 1, 8.0),     # peaky logits: exercises the online max rescale
    (1, 1000, 512, 2, 1.0),    # cross-attention shape (512 context tokens)
    (1, 1, 1, 1, 1.0),         # single query, single key
    (1, 129, 127, 1, 3.0),     # peaky, ragged
])
def test_attention(B, Sq, Skv, H, qmul):
    import torch
    D = H * 128
    q, k, v = _attn_case(B, Sq, Skv, H, qmul)
    o = torch.empty((B * Sq, D), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, H, Sq), dtype=torch.float32, device="cuda")
    dit.dit_attention(dev_bf16(q), dev_bf16(k), dev_bf16(v), o, B, Sq, Skv, H, lse=lse)
    qf, kf, vf = (synth.bf16_bits_to_f64(t) for t in (q, k, v))
    got = host_f64(o).reshape(B, Sq, D)
    lg = lse.cpu().double().numpy()
    for b in range(B):
        qs, ks, vs = qf[b * Sq:(b + 1) * Sq], kf[b * Skv:(b + 1) * Skv], vf[b * Skv:(b + 1) * Skv]
        ref = O.attention(qs, ks, vs, H)
        # Near-uniform softmax (qmul 1): the stated bound.  Peaky logits
        # (qmul 3, 8): a few keys dominate each row, so the largest outputs sit
        # near max|v| while averaging keeps RMS small; such an element carries
        # its own bf16 rounding (<= 2^-9 relative) plus the bf16 rounding of P
        # that the tensor-core PV product needs (<= 2^-9 relative per term),
        # hence the derived bound 3e-2 * RMS + 2^-7 * max|ref| for those cases
        # only.  rel L2 keeps 1e-2 and must also stay within 2x the error of
        # the exact result merely rounded to bf16 (+1e-3).
        rms = np.sqrt(np.mean(ref ** 2))
        frac = 3e-2 if qmul == 1.0 else 3e-2 + 2.0 ** -7 * np.abs(ref).max() / rms
        parity(got[b], ref, f"attention b={b}", max_abs_frac=frac)
        ref_b = synth.bf16_bits_to_f64(synth.f32_to_bf16_bits(ref.astype(np.float32)))
        floor = np.linalg.norm(ref_b - ref) / np.linalg.norm(ref)
        assert np.linalg.norm(got[b] - ref) / np.linalg.norm(ref) <= 2 * floor + 1e-3
        ref_lse = O.attention_lse(qs, ks, H)
        assert np.abs(lg[b] - ref_lse).max() < 1e-3 * max(1.0, np.abs(ref_lse).max())
    assert_no_device_error()


def test_attention_strided_views_in_packed_buffer():
    """q, k, v as column slices of one [S, 3D] buffer; o into a wider buffer."""
    import torch
    S, H = 200, 2
    D = H * 128
    qkv = synth.normal_bf16(7, "qkv", (S, 3 * D))
    d = dev_bf16(qkv)
    cat = torch.zeros((S, D + 512), dtype=torch.bfloat16, device="cuda")
    dit.dit_attention(d[:, :D], d[:, D:2 * D], d[:, 2 * D:], cat[:, :D], 1, S, S, H)
    f = synth.bf16_bits_to_f64(qkv)
    parity(host_f64(cat[:, :D]), O.attention(f[:, :D], f[:, D:2 * D], f[:, 2 * D:], H), "attention packed")
    assert torch.count_nonzero(cat[:, D:]) == 0


# ---------------------------------------------------------------- sequence-parallel pieces

@pytest.mark.parametrize("n,B,S,H", [(2, 1, 300, 3), (5, 2, 77, 2), (8, 1, 4608 // 8, 24)])
def test_attention_merge_matches_oracle(n, B, S, H):
    """Merge of n bf16 partial results with their fp32 lse against the fp64
    merge of the same inputs; in place into the first part and its lse."""
    import torch
    D = H * 128
    r = np.random.default_rng(n)
    parts = [synth.normal_bf16(20 + j, f"o{j}", (B * S, D)) for j in range(n)]
    lses = [(r.standard_normal((B, H, S)) * 3.0 + j).astype(np.float32) for j in range(n)]
    dp = [dev_bf16(t) for t in parts]
    dl = [torch.from_numpy(x).cuda() for x in lses]
    o = torch.empty((B * S, D), dtype=torch.bfloat16, device="cuda")
    lo = torch.empty((B, H, S), dtype=torch.float32, device="cuda")
    dit.dit_attention_merge(dp, dl, o, lo, B, S, H)
    pf = [synth.bf16_bits_to_f64(t).reshape(B, S, D) for t in parts]
    got = host_f64(o).reshape(B, S, D)
    for b in range(B):
        ref, ref_lse = O.attention_merge([p[b] for p in pf], [x[b].astype(np.float64) for x in lses])
        parity(got[b], ref, f"merge b={b}")
        assert np.abs(lo[b].cpu().double().numpy() - ref_lse).max() < 1e-5 * max(1.0, np.abs(ref_lse).max())
    # in place: the running result of a ring
    dit.dit_attention_merge(dp, dl, dp[0], dl[0], B, S, H)
    assert torch.equal(dp[0], o) and torch.equal(dl[0], lo)
    assert_no_device_error()


def test_attention_merge_empty_parts():
    """Parts over empty key sets (lse = -inf): a fully empty part carries no
    weight, and rows whose every part is empty give o = 0 and lse = -inf
    rather than NaN, as in the oracle's merge."""
    import torch
    B, S, H = 1, 50, 3
    D = H * 128
    r = np.random.default_rng(11)
    parts = [synth.normal_bf16(40 + j, f"e{j}", (S, D)) for j in range(3)]
    lses = [(r.standard_normal((B, H, S)) * 2.0).astype(np.float32) for _ in range(3)]
    lses[1][:] = -np.inf  # part 1 covers no keys at all
    for j in (0, 2):  # rows 7 and 31 of head 1 have no keys in any part
        lses[j][0, 1, [7, 31]] = -np.inf
    dp = [dev_bf16(t) for t in parts]
    dl = [torch.from_numpy(x).cuda() for x in lses]
    o = torch.empty((S, D), dtype=torch.bfloat16, device="cuda")
    lo = torch.empty((B, H, S), dtype=torch.float32, device="cuda")
    dit.dit_attention_merge(dp, dl, o, lo, B, S, H)
    torch.cuda.synchronize()
    pf = [synth.bf16_bits_to_f64(t) for t in parts]
    ref, ref_lse = O.attention_merge(pf, [x[0].astype(np.float64) for x in lses])
    got = host_f64(o)
    assert np.all(np.isfinite(got))
    gl = lo[0].cpu().double().numpy()
    assert np.array_equal(np.isneginf(gl), np.isneginf(ref_lse))
    fin = np.isfinite(ref_lse)
    assert np.abs(gl[fin] - ref_lse[fin]).max() < 1e-5 * max(1.0, np.abs(ref_lse[fin]).max())
    empty_cols = got[[7, 31]][:, 128:256]
    assert np.all(empty_cols == 0)
    parity(got, ref, "merge with empty parts")
    assert_no_device_error()


def test_ring_schedule_on_one_gpu_equals_full_attention():
    """The arithmetic of one rank's ring hops on one GPU: attention of the
    queries against each of 4 key/value shards (uneven tail), merged hop by
    hop into the running result, equals attention over all keys."""
    import torch
    S, H = 640, 4
    D = H * 128
    q, k, v = (synth.normal_bf16(60 + i, n, (S, D)) for i, n in enumerate("qkv"))
    dq, dk, dv = dev_bf16(q), dev_bf16(k), dev_bf16(v)
    cuts = [0, 128, 300, 512, 640]
    o = torch.empty((S, D), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((1, H, S), dtype=torch.float32, device="cuda")
    part = torch.empty_like(o)
    lpart = torch.empty_like(lse)
    for j, (a, b) in enumerate(zip(cuts, cuts[1:])):
        if j == 0:
            dit.dit_attention(dq, dk[a:b], dv[a:b], o, 1, S, b - a, H, lse=lse)
        else:
            dit.dit_attention(dq, dk[a:b], dv[a:b], part, 1, S, b - a, H, lse=lpart)
            dit.dit_attention_merge([o, part], [lse, lpart], o, lse, 1, S, H)
    qf, kf, vf = (synth.bf16_bits_to_f64(t) for t in (q, k, v))
    ref = O.attention(qf, kf, vf, H)
    rms = np.sqrt(np.mean(ref ** 2))
    # each hop's output and the merge round to bf16: four roundings of <= 2^-9
    parity(host_f64(o), ref, "ring on one GPU", max_abs_frac=3e-2 + 4 * 2.0 ** -9 * np.abs(ref).max() / rms)
    ref_lse = O.attention_lse(qf, kf, H)
    assert np.abs(lse[0].cpu().double().numpy() - ref_lse).max() < 1e-3 * max(1.0, np.abs(ref_lse).max())
    assert_no_device_error()


@pytest.mark.parametrize("cuts", [(0, 256, 512), (0, 100, 333, 576, 600), (0, 577)])
def test_attention_accumulate_over_key_splits(cuts):
    """dit_attention_accumulate folds the attention over one more key set into
    a running (o, lse): started from lse = -inf it equals dit_attention bit
    for bit, and accumulating over uneven key splits gives the attention over
    all keys (fp64 oracle) and its log-sum-exp.  Each step rounds the running
    output to bf16: max abs <= 3e-2 RMS + (steps) 2^-9 max|ref|."""
    import torch
    H, Sq = 3, 300
    D = H * 128
    Skv = cuts[-1]
    q, k, v = _attn_case(1, Sq, Skv, H, 2.0, seed=9)
    dq, dk, dv = dev_bf16(q), dev_bf16(k), dev_bf16(v)
    o = torch.zeros((Sq, D), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((1, H, Sq), float("-inf"), dtype=torch.float32, device="cuda")
    plain = torch.empty_like(o)
    plain_lse = torch.empty_like(lse)
    a, b = cuts[0], cuts[1]
    dit.dit_attention(dq, dk[a:b], dv[a:b], plain, 1, Sq, b - a, H, lse=plain_lse)
    dit.dit_attention_accumulate(dq, dk[a:b], dv[a:b], o, lse, 1, Sq, b - a, H)
    torch.cuda.synchronize()
    assert torch.equal(o, plain) and torch.equal(lse, plain_lse)
    for a, b in zip(cuts[1:], cuts[2:]):
        dit.dit_attention_accumulate(dq, dk[a:b], dv[a:b], o, lse, 1, Sq, b - a, H)
    torch.cuda.synchronize()
    qf, kf, vf = (synth.bf16_bits_to_f64(t) for t in (q, k, v))
    ref = O.attention(qf, kf, vf, H)
    rms = np.sqrt(np.mean(ref ** 2))
    steps = len(cuts) - 1
    parity(host_f64(o), ref, "accumulated attention",
           max_abs_frac=3e-2 + steps * 2.0 ** -9 * np.abs(ref).max() / rms)
    ref_lse = O.attention_lse(qf, kf, H)
    assert np.abs(lse[0].cpu().double().numpy() - ref_lse).max() < 1e-3 * max(1.0, np.abs(ref_lse).max())
    assert_no_device_error()


@pytest.mark.parametrize("B,Sq,Skv,H,n_split", [
    (1, 300, 600, 3, 2),    # 5 key tiles: parts of 3 + 2 tiles, ragged last tile
    (1, 576, 4608, 2, 2),   # one rank of a CP = 8 ring, all shards at once
    (2, 130, 1000, 2, 3),   # batch 2, three parts, ragged query and key tails
    (1, 200, 900, 2, 4),    # 8 tiles in four parts of two
    (1, 100, 100, 2, 4),    # one key tile: no split, no workspace needed
])
def test_attention_split_matches_oracle(B, Sq, Skv, H, n_split):
    """dit_attention_split cuts the keys into parts computed by separate CTAs
    of one launch and merges them by log-sum-exp: the result is the attention
    over all keys (fp64 oracle) with its log-sum-exp.  Each part is rounded to
    bf16 before the merge rounds once more: max abs <= 3e-2 RMS + 2 x 2^-9
    max|ref|."""
    import torch
    D = H * 128
    q, k, v = _attn_case(B, Sq, Skv, H, 2.0, seed=21)
    dq, dk, dv = dev_bf16(q), dev_bf16(k), dev_bf16(v)
    o = torch.empty((B * Sq, D), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, H, Sq), dtype=torch.float32, device="cuda")
    nbytes = dit.dit_attention_split_workspace(B, Sq, H, n_split)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    dit.dit_attention_split(dq, dk, dv, o, B, Sq, Skv, H, n_split, ws, lse=lse)
    torch.cuda.synchronize()
    qf, kf, vf = (synth.bf16_bits_to_f64(t) for t in (q, k, v))
    got = host_f64(o)
    for b in range(B):
        rows = slice(b * Sq, (b + 1) * Sq)
        kr = slice(b * Skv, (b + 1) * Skv)
        ref = O.attention(qf[rows], kf[kr], vf[kr], H)
        rms = np.sqrt(np.mean(ref ** 2))
        parity(got[rows], ref, f"split attention, batch {b}",
               max_abs_frac=3e-2 + 2 * 2.0 ** -9 * np.abs(ref).max() / rms)
        ref_lse = O.attention_lse(qf[rows], kf[kr], H)
        assert np.abs(lse[b].cpu().double().numpy() - ref_lse).max() < 1e-3 * max(1.0, np.abs(ref_lse).max())
    assert_no_device_error()


def test_attention_split_accumulates_like_a_ring():
    """A ring over three uneven key shards with two parts per step: the first
    step writes the running result, the later ones merge into it
    (accumulate = 1); the result is the attention over all keys."""
    import torch
    H, Sq = 2, 256
    D = H * 128
    cuts = (0, 700, 1100, 1800)
    q, k, v = _attn_case(1, Sq, cuts[-1], H, 2.0, seed=23)
    dq, dk, dv = dev_bf16(q), dev_bf16(k), dev_bf16(v)
    o = torch.empty((Sq, D), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((1, H, Sq), dtype=torch.float32, device="cuda")
    ws = torch.empty(dit.dit_attention_split_workspace(1, Sq, H, 2), dtype=torch.uint8, device="cuda")
    for i, (a, b) in enumerate(zip(cuts, cuts[1:])):
        dit.dit_attention_split(dq, dk[a:b], dv[a:b], o, 1, Sq, b - a, H, 2, ws, lse=lse, accumulate=i > 0)
    torch.cuda.synchronize()
    qf, kf, vf = (synth.bf16_bits_to_f64(t) for t in (q, k, v))
    ref = O.attention(qf, kf, vf, H)
    rms = np.sqrt(np.mean(ref ** 2))
    # each step: the parts and the running result are rounded once more
    parity(host_f64(o), ref, "split ring", max_abs_frac=3e-2 + 6 * 2.0 ** -9 * np.abs(ref).max() / rms)
    ref_lse = O.attention_lse(qf, kf, H)
    assert np.abs(lse[0].cpu().double().numpy() - ref_lse).max() < 1e-3 * max(1.0, np.abs(ref_lse).max())
    assert_no_device_error()


def test_attention_split_accumulates_into_a_strided_result():
    """The running result of a ring step may be a column block of a wider
    buffer (the block's [attn | mlp] concat, row stride D + M): split parts
    (row stride D) and the running result (its own stride) merge into it,
    and the columns beside it are left alone."""
    import torch
    H, Sq = 2, 300
    D = H * 128
    W = D + 512  # concat row: attention columns, then other columns
    cuts = (0, 640, 1000)
    q, k, v = _attn_case(1, Sq, cuts[-1], H, 1.5, seed=29)
    dq, dk, dv = dev_bf16(q), dev_bf16(k), dev_bf16(v)
    cat = torch.full((Sq, W), 7.0, dtype=torch.bfloat16, device="cuda")
    o = cat[:, :D]
    lse = torch.empty((1, H, Sq), dtype=torch.float32, device="cuda")
    ws = torch.empty(dit.dit_attention_split_workspace(1, Sq, H, 3), dtype=torch.uint8, device="cuda")
    for i, (a, b) in enumerate(zip(cuts, cuts[1:])):
        dit.dit_attention_split(dq, dk[a:b], dv[a:b], o, 1, Sq, b - a, H, 3, ws, lse=lse, accumulate=i > 0)
    torch.cuda.synchronize()
    assert bool((cat[:, D:] == 7.0).all())
    qf, kf, vf = (synth.bf16_bits_to_f64(t) for t in (q, k, v))
    ref = O.attention(qf, kf, vf, H)
    rms = np.sqrt(np.mean(ref ** 2))
    parity(host_f64(o.contiguous()), ref, "split ring into a strided result",
           max_abs_frac=3e-2 + 4 * 2.0 ** -9 * np.abs(ref).max() / rms)
    assert_no_device_error()


def test_sequence_parallel_drivers_with_cuda_kernels_one_rank():
    """ring_attention and ulysses_attention with their default CUDA local
    operations in a one-rank NCCL group (no transfer; the multi-rank
    schedules are checked on CPU ranks)."""
    import datetime
    import socket
    import torch
    import torch.distributed as dist
    from diffusion_transformer_block_flux_b200 import sequence_parallel as sp
    sock = socket.socket()
    sock.bind(("127.0.0.1", 0))
    port = sock.getsockname()[1]
    sock.close()
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60))
    try:
        S, H = 256, 2
        D = H * 128
        q, k, v = (synth.normal_bf16(70 + i, n, (S, D)) for i, n in enumerate("qkv"))
        dq, dk, dv = dev_bf16(q), dev_bf16(k), dev_bf16(v)
        ref = torch.empty((S, D), dtype=torch.bfloat16, device="cuda")
        dit.dit_attention(dq, dk, dv, ref, 1, S, S, H)
        o_ring = torch.empty_like(ref)
        sp.ring_attention(dq, dk, dv, o_ring, H, key_splits=1)
        o_uly = torch.empty_like(ref)
        sp.ulysses_attention(dq, dk, dv, o_uly, H)
        # the plan's default for so few query tiles cuts the keys (dit_attention_split)
        o_split = torch.empty_like(ref)
        sp.ring_attention(dq, dk, dv, o_split, H)
        torch.cuda.synchronize()
        assert torch.equal(o_ring, ref) and torch.equal(o_uly, ref)
        assert sp.auto_key_splits(S, H, "cuda") > 1
        qf, kf, vf = (synth.bf16_bits_to_f64(t) for t in (q, k, v))
        oref = O.attention(qf, kf, vf, H)
        rms = np.sqrt(np.mean(oref ** 2))
        parity(host_f64(o_split), oref, "ring with split keys",
               max_abs_frac=3e-2 + 2 * 2.0 ** -9 * np.abs(oref).max() / rms)
    finally:
        dist.destroy_process_group()
    assert_no_device_error()


@pytest.mark.parametrize("mode", ["ring", "ulysses"])
def test_sequence_parallel_block_one_rank_equals_block_and_graph_replays_it(mode):
    """The sequence-parallel single-stream block (static buffers, CUDA
    kernels) in a one-rank NCCL group runs the block's five kernels on the
    same inputs, so it equals dit_single_block_fwd bit for bit; captured into a
    CUDA graph (the Ulysses all-to-alls included), a replay gives the same bits
    again.  The multi-rank schedules are checked on CPU ranks."""
    import datetime
    import socket
    import torch
    import torch.distributed as dist
    from diffusion_transformer_block_flux_b200 import sequence_parallel as sp
    sock = socket.socket()
    sock.bind(("127.0.0.1", 0))
    port = sock.getsockname()[1]
    sock.close()
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60), device_id=torch.device("cuda", 0))
    graph = None
    try:
        s = synth.TINY
        wb = synth.single_block_weights(s, bias_std=synth.TEST_BIAS_STD, norm_scale_std=synth.TEST_NORM_SCALE_STD)
        ab = synth.block_activations(s)
        w = dev_tree(wb)
        x = dev_bf16(ab["x"])
        vec = dev_bf16(ab["vec"]).reshape(1, -1)
        rope = torch.empty((s.S, 64, 2), dtype=torch.float32, device="cuda")
        dit.dit_rope_table(torch.from_numpy(ab["ids"]).cuda(), (8, 28, 28), 10000.0, rope)
        cfg = dit.block_cfg(1, s.S, s.D, s.H, s.M)
        ws = torch.empty(dit.dit_single_block_workspace(cfg), dtype=torch.uint8, device="cuda")
        ref = torch.empty_like(x)
        dit.dit_single_block_fwd(cfg, dit.single_weights(w), x, vec, rope, ref, ws)
        blk = sp.SequenceParallelSingleBlock(s.S, s.D, s.H, s.M, "cuda", mode=mode, key_splits=1)
        out = torch.empty_like(x)
        blk.forward(w, x, vec, rope, out)
        torch.cuda.synchronize()
        assert torch.equal(out, ref)
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            blk.forward(w, x, vec, rope, out)  # warm-up on the capture stream
        torch.cuda.current_stream().wait_stream(side)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            blk.forward(w, x, vec, rope, out)
        out.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, ref)
        if mode == "ring":
            # the plan's default for so few query tiles cuts the keys
            # (dit_attention_split into the strided concat buffer): the oracle's
            # block within the block tolerance
            assert sp.auto_key_splits(s.S, s.H, "cuda") > 1
            blk2 = sp.SequenceParallelSingleBlock(s.S, s.D, s.H, s.M, "cuda", mode=mode)
            out2 = torch.empty_like(x)
            blk2.forward(w, x, vec, rope, out2)
            torch.cuda.synchronize()
            f = synth.to_f64(ab)
            oref = O.single_block(f["x"], f["vec"], f["ids"], synth.to_f64(wb), s.H)
            parity(host_f64(out2), oref, "sequence-parallel block, keys split")
    finally:
        del graph  # a graph holding NCCL work is released before the group
        dist.destroy_process_group()
    assert_no_device_error()


# ---------------------------------------------------------------- failure detection

def test_selftest_wait_times_out_and_reports():
    """A wait on a barrier nothing arrives on ends after its limit; the error
    word reports a timeout from the self-test site; the context stays usable."""
    import torch
    dit.dit_clear_device_error()
    dit.dit_selftest_wait_timeout(50_000_000)  # 50 ms
    st, code = dit.dit_get_device_error()
    assert st == dit.DIT_ERR_TIMEOUT
    assert code & 0xFF == dit.DIT_ERR_TIMEOUT and (code >> 8) == 1
    dit.dit_clear_device_error()
    assert dit.dit_get_device_error() == (0, 0)
    x = torch.ones(4, device="cuda")
    assert float((x * 2).sum()) == 8.0
