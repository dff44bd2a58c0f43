"""Pins for the fp64 oracle: invariants, closed forms, library special cases and
brute force on tiny inputs.  Each pin is chosen so that a plausible slip in the
oracle (a dropped term, a wrong sign, index or transposed operand) fails it.
CPU only."""
import cmath
import json
import math
import os
import statistics

import numpy as np
import pytest

from oracle import dit_oracle as O
from diffusion_transformer_block_flux_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rng(seed=0):
    return np.random.default_rng(seed)


# ---------------------------------------------------------------- elementwise

def test_silu_odd_identity_and_limits():
    x = rng().standard_normal(1000) * 5
    # x*sig(x) - (-x)*sig(-x) = x (sig(x) + sig(-x)) = x
    np.testing.assert_allclose(O.silu(x) - O.silu(-x), x, rtol=0, atol=1e-12)
    assert O.silu(0.0) == 0.0
    assert abs(O.silu(40.0) - 40.0) < 1e-12
    assert abs(O.silu(-40.0)) < 1e-12


def test_gelu_tanh_identity_and_erf_bound():
    u = np.linspace(-8, 8, 2001)
    # 0.5u(1+tanh z(u)) - 0.5(-u)(1+tanh z(-u)) = u since z is odd
    np.testing.assert_allclose(O.gelu_tanh(u) - O.gelu_tanh(-u), u, atol=1e-12)
    exact = np.array([0.5 * x * (1 + math.erf(x / math.sqrt(2))) for x in u])
    # the tanh form's approximation error is below 5e-4 everywhere
    assert np.abs(O.gelu_tanh(u) - exact).max() < 1e-3
    assert O.gelu_tanh(0.0) == 0.0
    assert abs(O.gelu_tanh(12.0) - 12.0) < 1e-12


# ---------------------------------------------------------------- LayerNorm

def test_layer_norm_moments():
    x = rng(1).standard_normal((64, 384)) * 3 + 2
    eps = 1e-6
    n = O.layer_norm(x, eps)
    var = x.var(axis=1)
    np.testing.assert_allclose(n.mean(axis=1), 0, atol=1e-12)
    np.testing.assert_allclose(n.var(axis=1), var / (var + eps), rtol=1e-12)


def test_layer_norm_constant_row_and_statistics_module():
    assert np.all(O.layer_norm(np.full((2, 8), 3.5)) == 0)
    row = [1.0, 4.0, -2.0, 0.5, 7.0]
    mu = statistics.fmean(row)
    sd = math.sqrt(statistics.pvariance(row) + 1e-6)
    np.testing.assert_allclose(O.layer_norm(np.array([row]))[0],
                               [(r - mu) / sd for r in row], rtol=1e-14)


def test_modulate_identity_and_affine():
    n = rng(2).standard_normal((4, 16))
    z = np.zeros(16)
    np.testing.assert_array_equal(O.modulate(n, z, z), n)
    sh, sc = rng(3).standard_normal(16), rng(4).standard_normal(16)
    y = O.modulate(n, sh, sc)
    # elementwise affine in n with slope 1+scale and offset shift
    np.testing.assert_allclose(O.modulate(n + 1, sh, sc) - y, np.broadcast_to(1 + sc, y.shape), atol=1e-12)
    np.testing.assert_allclose(O.modulate(np.zeros_like(n), sh, sc), np.broadcast_to(sh, y.shape))


# ---------------------------------------------------------------- linear / adaLN

def test_linear_brute_force_and_identity():
    x = rng(5).standard_normal((3, 4))
    W = rng(6).standard_normal((5, 4))
    b = rng(7).standard_normal(5)
    ref = [[sum(x[i, k] * W[j, k] for k in range(4)) + b[j] for j in range(5)] for i in range(3)]
    np.testing.assert_allclose(O.linear(x, W, b), ref, rtol=1e-13)
    np.testing.assert_array_equal(O.linear(x, np.eye(4)), x)


def test_adaln_chunk_order_and_silu_first():
    D = 8
    b = np.concatenate([np.full(D, 1.0), np.full(D, 2.0), np.full(D, 3.0)])
    shift, scale, gate = O.adaln_modulation(rng(8).standard_normal(D), np.zeros((3 * D, D)), b, 3)
    assert np.all(shift == 1) and np.all(scale == 2) and np.all(gate == 3)
    # one-hot weight picks silu(vec[j])
    vec = np.array([0.0, -1.0, 2.0, 0.0, 0.0, 0.0, 0.0, 0.0])
    W = np.zeros((3 * D, D))
    W[D + 5, 2] = 1.0  # scale[5] <- silu(vec[2])
    _, scale, _ = O.adaln_modulation(vec, W, np.zeros(3 * D), 3)
    assert abs(scale[5] - 2.0 / (1.0 + math.exp(-2.0))) < 1e-15
    assert np.count_nonzero(scale) == 1


# ---------------------------------------------------------------- RMSNorm

def test_rms_norm_heads_unit_rms():
    eps = 1e-6
    x = rng(9).standard_normal((10, 3 * 128)) * 4
    y = O.rms_norm_heads(x, np.ones(128), 3, eps).reshape(10, 3, 128)
    ms = (x.reshape(10, 3, 128) ** 2).mean(-1)
    np.testing.assert_allclose(np.sqrt((y ** 2).mean(-1)), np.sqrt(ms / (ms + eps)), rtol=1e-12)
    # per-dimension scale multiplies the normalised value
    s = rng(10).standard_normal(128)
    y2 = O.rms_norm_heads(x, s, 3, eps).reshape(10, 3, 128)
    np.testing.assert_allclose(y2, y * s, rtol=1e-12, atol=1e-14)
    # heads are independent: scaling one head's input leaves the others alone
    x3 = x.copy().reshape(10, 3, 128)
    x3[:, 1] *= 7
    y3 = O.rms_norm_heads(x3.reshape(10, -1), np.ones(128), 3, eps).reshape(10, 3, 128)
    np.testing.assert_allclose(y3[:, 0], y[:, 0])
    np.testing.assert_allclose(y3[:, 1], y[:, 1], rtol=1e-6)


# ---------------------------------------------------------------- RoPE

AX = (16, 56, 56)


def test_rope_identity_at_origin_and_norm_preserved():
    ids = synth.flux_ids(4, 3, 5)
    x = rng(11).standard_normal((ids.shape[0], 2 * 128))
    phi = O.rope_angles(ids, AX)
    y = O.apply_rope(x, phi, 2)
    np.testing.assert_array_equal(y[:4], x[:4])  # text tokens at (0,0,0)
    pn = lambda a: np.hypot(a.reshape(a.shape[0], -1, 2)[..., 0], a.reshape(a.shape[0], -1, 2)[..., 1])
    np.testing.assert_allclose(pn(y), pn(x), rtol=1e-12)


def test_rope_frequency_structure():
    ids = np.array([[0, 0, 1], [0, 1, 0], [1, 0, 0]])
    phi = O.rope_angles(ids, AX, 10000.0)
    # (0,0,1): only the w axis (pairs 36..63) turns; its first pair by 1 rad
    assert np.all(phi[0, :36] == 0) and phi[0, 36] == 1.0
    # (0,1,0): only the h axis (pairs 8..35)
    assert np.all(phi[1, :8] == 0) and np.all(phi[1, 36:] == 0) and phi[1, 8] == 1.0
    # (1,0,0): only the t axis (pairs 0..7)
    assert np.all(phi[2, 8:] == 0) and phi[2, 0] == 1.0
    for row, lo, n in ((0, 36, 28), (1, 8, 28), (2, 0, 8)):
        w = phi[row, lo:lo + n]
        ratio = w[1:] / w[:-1]
        np.testing.assert_allclose(ratio, ratio[0], rtol=1e-12)  # geometric
        # a quarter of the axis dim in, the frequency is theta^(-1/2)
        np.testing.assert_allclose(w[n // 2], 10000.0 ** -0.5, rtol=1e-12)
        assert np.all(np.diff(w) < 0)


def test_rope_matches_complex_multiplication():
    ids = np.array([[2, 5, 7]])
    x = rng(12).standard_normal((1, 128))
    phi = O.rope_angles(ids, AX)
    y = O.apply_rope(x, phi, 1)
    for p in (0, 3, 8, 20, 36, 63):
        z = complex(x[0, 2 * p], x[0, 2 * p + 1]) * cmath.exp(1j * phi[0, p])
        assert abs(z.real - y[0, 2 * p]) < 1e-12 and abs(z.imag - y[0, 2 * p + 1]) < 1e-12


def test_rope_relative_position_property():
    # rope(q, m) . rope(k, n) depends only on m - n: shifting every id by a
    # constant leaves all logits unchanged.
    ids = synth.flux_ids(0, 4, 6)
    q = rng(13).standard_normal((ids.shape[0], 128))
    k = rng(14).standard_normal((ids.shape[0], 128))
    a = O.apply_rope(q, O.rope_angles(ids, AX), 1) @ O.apply_rope(k, O.rope_angles(ids, AX), 1).T
    ids2 = ids + np.array([3, 11, -5])
    b = O.apply_rope(q, O.rope_angles(ids2, AX), 1) @ O.apply_rope(k, O.rope_angles(ids2, AX), 1).T
    np.testing.assert_allclose(a, b, rtol=1e-9, atol=1e-9)


# ---------------------------------------------------------------- attention

def brute_attention(q, k, v, scale):
    out = []
    for i in range(len(q)):
        logits = [scale * sum(a * b for a, b in zip(q[i], k[j])) for j in range(len(k))]
        m = max(logits)
        e = [math.exp(l - m) for l in logits]
        s = sum(e)
        out.append([sum(e[j] * v[j][c] for j in range(len(k))) / s for c in range(len(v[0]))])
    return np.array(out)


def test_attention_brute_force_tiny():
    q = rng(15).standard_normal((3, 8))
    k = rng(16).standard_normal((5, 8))
    v = rng(17).standard_normal((5, 8))
    got = O.attention(q, k, v, n_heads=2)
    for h in range(2):
        sl = slice(4 * h, 4 * h + 4)
        np.testing.assert_allclose(got[:, sl], brute_attention(q[:, sl], k[:, sl], v[:, sl], 0.5),
                                   rtol=1e-12)


def test_attention_special_cases():
    d = 128
    q = rng(18).standard_normal((4, d))
    v = rng(19).standard_normal((1, d))
    np.testing.assert_allclose(O.attention(q, rng(20).standard_normal((1, d)), v, 1),
                               np.repeat(v, 4, 0), rtol=1e-13)
    kk = np.repeat(rng(21).standard_normal((1, d)), 6, 0)
    vv = rng(22).standard_normal((6, d))
    np.testing.assert_allclose(O.attention(q, kk, vv, 1), np.repeat(vv.mean(0, keepdims=True), 4, 0),
                               rtol=1e-12)
    # one key aligned with the query with a huge logit takes all the weight
    k3 = rng(23).standard_normal((6, d)) * 0.01
    k3[4] = q[0] / np.dot(q[0], q[0]) * 50 * math.sqrt(d)
    np.testing.assert_allclose(O.attention(q[:1], k3, vv, 1)[0], vv[4], atol=1e-12)


def test_attention_key_permutation_and_rows():
    q = rng(24).standard_normal((7, 256))
    k = rng(25).standard_normal((9, 256))
    v = rng(26).standard_normal((9, 256))
    p = rng(27).permutation(9)
    np.testing.assert_allclose(O.attention(q, k, v, 2), O.attention(q, k[p], v[p], 2), rtol=1e-12)
    np.testing.assert_allclose(O.attention(q, k, v, 2, rows=[5, 1]), O.attention(q, k, v, 2)[[5, 1]],
                               rtol=1e-13)


def test_attention_lse_brute_force():
    q = rng(28).standard_normal((3, 8))
    k = rng(29).standard_normal((4, 8))
    lse = O.attention_lse(q, k, 1)
    for i in range(3):
        ref = math.log(sum(math.exp(np.dot(q[i], k[j]) / math.sqrt(8)) for j in range(4)))
        assert abs(lse[0, i] - ref) < 1e-12


# ---------------------------------------------------------------- blocks

def _tiny_shape():
    return synth.BlockShape("t", 8, 2, 4, 256, 2, 512)


def test_single_block_zero_modulation_is_identity():
    s = _tiny_shape()
    w = synth.to_f64(synth.single_block_weights(s, zero_mod=True))
    a = synth.to_f64(synth.block_activations(s))
    out = O.single_block(a["x"], a["vec"], a["ids"], w, s.H)
    np.testing.assert_array_equal(out, a["x"])


def test_single_block_rows_subset_and_permutation_equivariance():
    s = _tiny_shape()
    w = synth.to_f64(synth.single_block_weights(s))
    a = synth.to_f64(synth.block_activations(s))
    full = O.single_block(a["x"], a["vec"], a["ids"], w, s.H)
    rows = np.array([0, 5, 9, 15])
    np.testing.assert_allclose(O.single_block(a["x"], a["vec"], a["ids"], w, s.H, rows=rows),
                               full[rows], rtol=1e-12, atol=1e-12)
    perm = rng(30).permutation(s.S)
    outp = O.single_block(a["x"][perm], a["vec"], a["ids"][perm], w, s.H)
    np.testing.assert_allclose(outp, full[perm], rtol=1e-10, atol=1e-10)
    # the block is not the identity for random modulation
    assert np.abs(full - a["x"]).max() > 1e-2


def test_double_block_zero_modulation_and_stream_swap():
    s = _tiny_shape()
    a = synth.to_f64(synth.double_block_activations(s))
    w0 = synth.to_f64(synth.double_block_weights(s, zero_mod=True))
    img, txt = O.double_block(a["img"], a["txt"], a["vec"], a["ids"], w0, s.H)
    np.testing.assert_array_equal(img, a["img"])
    np.testing.assert_array_equal(txt, a["txt"])
    w = synth.to_f64(synth.double_block_weights(s))
    n_txt = s.n_txt
    img1, txt1 = O.double_block(a["img"], a["txt"], a["vec"], a["ids"], w, s.H)
    # swap the streams' roles: weights, token sets and their ids
    ids_sw = np.concatenate([a["ids"][n_txt:], a["ids"][:n_txt]])
    img2, txt2 = O.double_block(a["txt"], a["img"], a["vec"], ids_sw,
                                {"txt": w["img"], "img": w["txt"]}, s.H)
    np.testing.assert_allclose(img2, txt1, rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(txt2, img1, rtol=1e-10, atol=1e-10)


def test_double_block_rows_subset():
    s = _tiny_shape()
    a = synth.to_f64(synth.double_block_activations(s))
    w = synth.to_f64(synth.double_block_weights(s))
    img, txt = O.double_block(a["img"], a["txt"], a["vec"], a["ids"], w, s.H)
    ri, rt = np.array([0, 3, 7]), np.array([1, 6])
    img_r, txt_r = O.double_block(a["img"], a["txt"], a["vec"], a["ids"], w, s.H, rows_img=ri, rows_txt=rt)
    np.testing.assert_allclose(img_r, img[ri], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(txt_r, txt[rt], rtol=1e-12, atol=1e-12)


def test_double_block_per_stream_independence_of_weights():
    """Changing the text stream's MLP weights leaves the image output alone
    (the streams only meet in attention, which precedes the MLP)."""
    s = _tiny_shape()
    a = synth.to_f64(synth.double_block_activations(s))
    w = synth.to_f64(synth.double_block_weights(s))
    img1, txt1 = O.double_block(a["img"], a["txt"], a["vec"], a["ids"], w, s.H)
    w["txt"]["W_mlp2"] = w["txt"]["W_mlp2"] * 3
    img2, txt2 = O.double_block(a["img"], a["txt"], a["vec"], a["ids"], w, s.H)
    np.testing.assert_array_equal(img1, img2)
    assert np.abs(txt1 - txt2).max() > 1e-3


def test_video_block_identity_and_rows():
    vs = synth.VideoShape("v", 2, 3, 4, 256, 2, 384, 5)
    w = synth.to_f64(synth.video_block_weights(vs))
    a = synth.to_f64(synth.video_activations(vs))
    full = O.video_block(a["x"], a["ctx"], a["vec"], a["ids"], w, vs.H)
    rows = np.array([1, 7, 23])
    np.testing.assert_allclose(O.video_block(a["x"], a["ctx"], a["vec"], a["ids"], w, vs.H, rows=rows),
                               full[rows], rtol=1e-12, atol=1e-12)
    w0 = dict(w)
    w0["W_mod"] = np.zeros_like(w["W_mod"])
    w0["W_co"] = np.zeros_like(w["W_co"])
    np.testing.assert_array_equal(O.video_block(a["x"], a["ctx"], a["vec"], a["ids"], w0, vs.H), a["x"])
    # cross attention alone: with zero modulation the block adds ctx attention only
    w1 = dict(w0)
    w1["W_co"] = w["W_co"]
    out1 = O.video_block(a["x"], a["ctx"], a["vec"], a["ids"], w1, vs.H)
    cq = O.linear(O.layer_norm(a["x"]), w["W_cq"], w["b_cq"])
    ckv = O.linear(a["ctx"], w["W_ckv"], w["b_ckv"])
    co = O.attention(cq, ckv[:, :256], ckv[:, 256:], vs.H)
    np.testing.assert_allclose(out1, a["x"] + O.linear(co, w["W_co"], w["b_co"]), rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- model / loop

def test_timestep_embedding_closed_forms():
    e0 = O.timestep_embedding(0.0)
    np.testing.assert_array_equal(e0, np.concatenate([np.ones(128), np.zeros(128)]))
    for t in (0.3, 1.0):
        e = O.timestep_embedding(t)
        np.testing.assert_allclose(e[:128] ** 2 + e[128:] ** 2, 1.0, rtol=1e-12)
        assert abs(e[0] - math.cos(1000 * t)) < 1e-12 and abs(e[128] - math.sin(1000 * t)) < 1e-12


def test_patchify_roundtrip_and_index_map():
    lat = rng(31).standard_normal((3, 4, 6))
    tok = O.patchify(lat)
    assert tok.shape == (6, 12)
    for h in range(2):
        for w_ in range(3):
            for c in range(3):
                for ph in range(2):
                    for pw in range(2):
                        assert tok[h * 3 + w_, c * 4 + ph * 2 + pw] == lat[c, 2 * h + ph, 2 * w_ + pw]
    np.testing.assert_array_equal(O.unpatchify(tok, 3, 2, 3), lat)


def _tiny_loop():
    b = synth.BlockShape("lt", 4, 2, 3, 256, 2, 256)
    return synth.loop_shape(b, 1, 1, 3, channels=2, txt_in=64)


def test_euler_constant_velocity_closed_form():
    ls = _tiny_loop()
    m = synth.to_f64(synth.model_weights(ls))
    inp = synth.to_f64(synth.loop_inputs(ls))
    m["W_out"] = np.zeros_like(m["W_out"])
    c = rng(32).standard_normal(m["b_out"].shape)
    m["b_out"] = c
    out = O.euler_sample(inp["latent"], inp["txt"], inp["ids"], m, ls.block.H, ls.steps)
    # sum of (t_{i+1} - t_i) over the schedule 1 -> 0 is -1
    tok = O.patchify(inp["latent"]) - c
    np.testing.assert_allclose(out, O.unpatchify(tok, 2, 2, 3), rtol=1e-12, atol=1e-12)


def test_step_cache_all_fresh_and_constant_velocity():
    ls = _tiny_loop()
    m = synth.to_f64(synth.model_weights(ls))
    inp = synth.to_f64(synth.loop_inputs(ls))
    base = O.euler_sample(inp["latent"], inp["txt"], inp["ids"], m, ls.block.H, ls.steps)
    all_fresh = O.euler_sample(inp["latent"], inp["txt"], inp["ids"], m, ls.block.H, ls.steps,
                               fresh=[1] * ls.steps)
    np.testing.assert_array_equal(base, all_fresh)
    # a constant velocity is reproduced exactly by both cache rules
    m["W_out"] = np.zeros_like(m["W_out"])
    c = rng(33).standard_normal(m["b_out"].shape)
    m["b_out"] = c
    for order in (0, 1):
        out = O.euler_sample(inp["latent"], inp["txt"], inp["ids"], m, ls.block.H, ls.steps,
                             fresh=[1, 1, 0], cache_order=order)
        tok = O.patchify(inp["latent"]) - c
        np.testing.assert_allclose(out, O.unpatchify(tok, 2, 2, 3), rtol=1e-12, atol=1e-12)


def test_step_cache_first_order_bookkeeping():
    """3 steps over t = 1, 2/3, 1/3 with steps 0, 1 fresh and step 2 cached:
    the prediction is v2 = v1 + (t2 - t1)(v1 - v0)/(t1 - t0) = 2 v1 - v0."""
    ls = _tiny_loop()
    m = synth.to_f64(synth.model_weights(ls))
    inp = synth.to_f64(synth.loop_inputs(ls))
    x0 = O.patchify(inp["latent"])
    v0 = O.flux_velocity(x0, inp["txt"], 1.0, inp["ids"], m, ls.block.H)
    x1 = x0 - v0 / 3
    v1 = O.flux_velocity(x1, inp["txt"], 2.0 / 3.0, inp["ids"], m, ls.block.H)
    x2 = x1 - v1 / 3
    x3 = x2 - (2 * v1 - v0) / 3
    got = O.euler_sample(inp["latent"], inp["txt"], inp["ids"], m, ls.block.H, 3, fresh=[1, 1, 0], cache_order=1)
    np.testing.assert_allclose(got, O.unpatchify(x3, 2, 2, 3), rtol=1e-10, atol=1e-12)
    got0 = O.euler_sample(inp["latent"], inp["txt"], inp["ids"], m, ls.block.H, 3, fresh=[1, 1, 0], cache_order=0)
    np.testing.assert_allclose(got0, O.unpatchify(x2 - v1 / 3, 2, 2, 3), rtol=1e-10, atol=1e-12)


def test_golden_flux_shapes():
    with open(os.path.join(GOLDEN, "flux_shapes.json")) as f:
        g = json.load(f)
    sb = g["single_block"]
    assert synth.FLUX.S == sb["S"] and synth.FLUX.D == sb["dim"]
    assert synth.FLUX.H == sb["heads"] and synth.FLUX.d == sb["head_dim"]
    assert synth.FLUX_LOOP.n_double + synth.FLUX_LOOP.n_single == g["model_blocks"]
    assert synth.FLUX_LOOP.steps == g["steps"]
    assert synth.FLUX.grid_h * 8 * 2 == g["image_px"]  # VAE /8 then 2x2 patches: 1024 -> 64
    assert synth.FLUX.H * synth.FLUX.d == synth.FLUX.D


def test_flops_model():
    f = O.single_block_flops(4608, 3072, 12288, 24)
    assert abs(f - 1.3047e12) / 1.3047e12 < 1e-3


def test_attention_merge_over_key_splits_is_full_attention():
    """Splitting the keys into disjoint sets and merging by log-sum-exp gives
    the attention over all keys (up to rounding), for uneven splits and a
    permuted order of the parts."""
    r = rng(41)
    H, d, Sq, Skv = 2, 8, 5, 23
    q, k, v = (r.standard_normal((n, H * d)) for n in (Sq, Skv, Skv))
    full = O.attention(q, k, v, H)
    full_lse = O.attention_lse(q, k, H)
    cuts = [0, 4, 5, 15, 23]
    outs = [O.attention(q, k[a:b], v[a:b], H) for a, b in zip(cuts, cuts[1:])]
    lses = [O.attention_lse(q, k[a:b], H) for a, b in zip(cuts, cuts[1:])]
    o, lse = O.attention_merge(outs[::-1], lses[::-1])
    np.testing.assert_allclose(o, full, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse, full_lse, rtol=1e-12, atol=1e-12)
    # one part: unchanged; a part with lse far below the others gets no weight
    o1, l1 = O.attention_merge(outs[:1], lses[:1])
    np.testing.assert_array_equal(o1, outs[0])
    o2, _ = O.attention_merge([outs[0], outs[1] + 1e6], [lses[0], lses[1] - 1e4])
    np.testing.assert_allclose(o2, outs[0], rtol=1e-12, atol=1e-9)
    # an empty key set (lse = log 0 = -inf) carries no weight: merging it changes nothing
    empty_o, empty_l = np.full_like(outs[0], 5.0), np.full_like(lses[0], -np.inf)
    o3, l3 = O.attention_merge([outs[0], empty_o, outs[1]], [lses[0], empty_l, lses[1]])
    o4, l4 = O.attention_merge([outs[0], outs[1]], [lses[0], lses[1]])
    np.testing.assert_array_equal(o3, o4)
    np.testing.assert_array_equal(l3, l4)
    # every part empty: the empty union, o = 0 and lse = -inf (no NaN)
    o5, l5 = O.attention_merge([empty_o, empty_o], [empty_l, empty_l])
    assert np.all(o5 == 0) and np.all(np.isneginf(l5))
    # rows may differ: only the row whose parts are all empty gets the empty result
    la, lb = lses[0].copy(), lses[1].copy()
    la[:, 2] = -np.inf
    lb[:, 2] = -np.inf
    o6, l6 = O.attention_merge([outs[0], outs[1]], [la, lb])
    assert np.all(o6[2] == 0) and np.all(np.isneginf(l6[:, 2]))
    np.testing.assert_array_equal(o6[[0, 1, 3, 4]], o4[[0, 1, 3, 4]])


def test_guidance_special_cases_and_bookkeeping():
    """Classifier-free guidance in the sampler: guidance 1 gives the
    conditional sampler, guidance 0 the unconditional one, equal texts make
    the guidance irrelevant, cfg_steps = 0 switches it off; two guided steps
    rebuilt by hand from four explicit model calls."""
    ls = _tiny_loop()
    m = synth.to_f64(synth.model_weights(ls))
    inp = synth.to_f64(synth.loop_inputs(ls))
    lat, txt, ids, H = inp["latent"], inp["txt"], inp["ids"], ls.block.H
    unc = rng(77).standard_normal(txt.shape)
    cond = O.euler_sample(lat, txt, ids, m, H, ls.steps)
    unco = O.euler_sample(lat, unc, ids, m, H, ls.steps)
    close = dict(rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(O.euler_sample(lat, txt, ids, m, H, ls.steps, txt_uncond=unc, guidance=1.0), cond, **close)
    np.testing.assert_allclose(O.euler_sample(lat, txt, ids, m, H, ls.steps, txt_uncond=unc, guidance=0.0), unco, **close)
    np.testing.assert_allclose(O.euler_sample(lat, txt, ids, m, H, ls.steps, txt_uncond=txt, guidance=4.0), cond, **close)
    np.testing.assert_allclose(O.euler_sample(lat, txt, ids, m, H, ls.steps, txt_uncond=unc, guidance=4.0,
                                              cfg_steps=0), cond, **close)
    g = 3.5
    x0 = O.patchify(lat)
    v0 = O.flux_velocity(x0, unc, 1.0, ids, m, H)
    v0 = v0 + g * (O.flux_velocity(x0, txt, 1.0, ids, m, H) - v0)
    x1 = x0 - v0 / 2
    v1 = O.flux_velocity(x1, txt, 0.5, ids, m, H)  # guidance only for the first step (cfg_steps = 1)
    x2 = x1 - v1 / 2
    got = O.euler_sample(lat, txt, ids, m, H, 2, txt_uncond=unc, guidance=g, cfg_steps=1)
    np.testing.assert_allclose(got, O.unpatchify(x2, 2, 2, 3), **close)


# ---------------------------------------------------------------- model forward (flux_velocity)

def _sig(z):
    """Logistic function written as (1 + tanh(z/2)) / 2: an expression
    independent of the oracle's z / (1 + e^-z)."""
    return 0.5 * (1.0 + math.tanh(0.5 * z))


def _ln_row(r, eps=1e-6):
    r = np.asarray(r, dtype=np.float64)
    return (r - statistics.fmean(r)) / math.sqrt(statistics.pvariance(r) + eps)


def _bare_model(D, cin, txt_in, t_dim=256):
    z = lambda *s: np.zeros(s)
    return {"W_img_in": z(D, cin), "b_img_in": z(D), "W_txt_in": z(D, txt_in), "b_txt_in": z(D),
            "W_t1": z(D, t_dim), "b_t1": z(D), "W_t2": z(D, D), "b_t2": z(D),
            "W_fmod": z(2 * D, D), "b_fmod": z(2 * D), "W_out": z(cin, D), "b_out": z(cin),
            "double": [], "single": []}


def test_flux_velocity_final_layer_order_time_mlp_and_img_in():
    """One-hot weights route single values through the top level of the model
    (the compile_graph page's eager forward, §3.1), with no blocks:
      time path: h = W_t1 emb + b_t1 picks emb[0] = cos(1000 t) (cos half
        first); vec = W_t2 silu(h) + b_t2 picks silu(h); the final adaLN adds
        silu(vec) to shift j: two SiLUs in a row;
      img_in: every image row is tok[t, 0] * u with u = (+1, -1, ...), whose
        LayerNorm is tok0 u / sqrt(tok0^2 + eps) in closed form;
      final layer: chunk 0 of W_fmod silu(vec) + b_fmod is the shift and chunk
        1 the scale: v = ((1 + scale) LN + shift) W_out^T + b_out.
    A swapped (shift, scale), a missing SiLU, or sin/cos in the other order
    changes the value."""
    D, H, C = 256, 2, 2
    cin, n_txt, gh, gw, tdim = 4 * C, 4, 2, 3, 256
    r = rng(61)
    m = _bare_model(D, cin, 16, tdim)
    u = np.array([1.0 if j % 2 == 0 else -1.0 for j in range(D)])
    m["W_img_in"][:, 0] = u
    i0, k, j, j1, f0, f1 = 5, 9, 17, 40, 3, 6
    m["W_t1"][i0, 0] = 1.0
    m["W_t2"][k, i0] = 1.0
    m["W_fmod"][j, k] = 1.0
    m["b_fmod"] = r.standard_normal(2 * D) * 0.5
    m["W_out"][f0, j] = 1.0
    m["W_out"][f1, j1] = 1.0
    m["b_out"] = r.standard_normal(cin)
    tok = r.standard_normal((gh * gw, cin))
    txt = r.standard_normal((n_txt, 16))
    ids = synth.flux_ids(n_txt, gh, gw)
    t = 0.37
    v = O.flux_velocity(tok, txt, t, ids, m, H)
    assert v.shape == (gh * gw, cin)
    c = math.cos(1000.0 * t)
    vec_k = c * _sig(c)
    s = vec_k * _sig(vec_k)  # silu(silu(cos(1000 t)))
    sh, sc = m["b_fmod"][:D], m["b_fmod"][D:]
    for ti in range(gh * gw):
        a = tok[ti, 0]
        ln = a * u / math.sqrt(a * a + 1e-6)
        assert abs(v[ti, f0] - ((1 + sc[j]) * ln[j] + sh[j] + s + m["b_out"][f0])) < 1e-12
        assert abs(v[ti, f1] - ((1 + sc[j1]) * ln[j1] + sh[j1] + m["b_out"][f1])) < 1e-12
        for f in range(cin):
            if f not in (f0, f1):
                assert v[ti, f] == m["b_out"][f]


def test_flux_velocity_text_joins_the_image_through_joint_attention():
    """One single-stream block whose attention is uniform (q = k = 0) and whose
    branch is o alone (v = LN(x), W2 = [I | 0], gate 1, scale = shift = 0):
    every token becomes x_t + mean_s LN(x_s) over the joint sequence, so the
    image velocity depends on txt_in(txt) through the mean.  Checked against
    the text and image embeddings written out with their biases, the joint
    mean over txt | img, and the final layer on the image rows only."""
    D, H, C = 256, 2, 2
    cin, n_txt, gh, gw, tin = 4 * C, 5, 2, 3, 16
    r = rng(62)
    m = _bare_model(D, cin, tin)
    m["W_img_in"] = r.standard_normal((D, cin))
    m["b_img_in"] = r.standard_normal(D)
    m["W_txt_in"] = r.standard_normal((D, tin)) * 0.3
    m["b_txt_in"] = r.standard_normal(D)
    picks = [7, 100, 255, 31, 0, 64, 128, 200]
    for f, jf in enumerate(picks):
        m["W_out"][f, jf] = 1.0
    Mh = 64
    W1 = np.zeros((3 * D + Mh, D))
    W1[2 * D:3 * D] = np.eye(D)  # v = y
    W2 = np.zeros((D, D + Mh))
    W2[:, :D] = np.eye(D)  # branch = o
    b_mod = np.concatenate([np.zeros(2 * D), np.ones(D)])  # shift 0, scale 0, gate 1
    m["single"] = [{"W_mod": np.zeros((3 * D, D)), "b_mod": b_mod, "W1": W1, "b1": np.zeros(3 * D + Mh),
                    "q_scale": np.ones(128), "k_scale": np.ones(128), "W2": W2, "b2": np.zeros(D)}]
    tok = r.standard_normal((gh * gw, cin))
    txt = r.standard_normal((n_txt, tin))
    ids = synth.flux_ids(n_txt, gh, gw)
    v = O.flux_velocity(tok, txt, 0.5, ids, m, H)
    te = [[sum(txt[s, i] * m["W_txt_in"][o, i] for i in range(tin)) + m["b_txt_in"][o] for o in range(D)]
          for s in range(n_txt)]
    ie = [[sum(tok[s, i] * m["W_img_in"][o, i] for i in range(cin)) + m["b_img_in"][o] for o in range(D)]
          for s in range(gh * gw)]
    lns = [_ln_row(row) for row in te + ie]
    mean = np.sum(lns, axis=0) / len(lns)
    for ti in range(gh * gw):
        y = _ln_row(np.asarray(ie[ti]) + mean)
        for f, jf in enumerate(picks):
            assert abs(v[ti, f] - y[jf]) < 1e-10
    # the text matters: another text gives another image velocity
    v2 = O.flux_velocity(tok, txt * 2 + 1, 0.5, ids, m, H)
    assert np.abs(v2 - v).max() > 1e-3


def test_flux_velocity_identity_blocks_leave_the_embedding():
    """Double and single blocks with zero modulation are the identity (gate 0),
    so the velocity equals that of the same model with no blocks, bit for bit:
    the double block's (img, txt) outputs go back to the right streams and the
    image rows are split off the joint sequence after the single blocks."""
    b = synth.BlockShape("vi", 5, 2, 3, 256, 2, 256)
    ls = synth.loop_shape(b, 2, 2, 1, channels=2, txt_in=64)
    m = synth.to_f64(synth.model_weights(ls, bias_std=0.1))
    zd = synth.to_f64(synth.double_block_weights(b, zero_mod=True, bias_std=0.1))
    zs = synth.to_f64(synth.single_block_weights(b, zero_mod=True, bias_std=0.1))
    inp = synth.to_f64(synth.loop_inputs(ls))
    tok = O.patchify(inp["latent"])
    bare = dict(m, double=[], single=[])
    ident = dict(m, double=[zd], single=[zs, zs])  # one double block: a swap of its outputs would stay
    v0 = O.flux_velocity(tok, inp["txt"], 0.8, inp["ids"], bare, b.H)
    v1 = O.flux_velocity(tok, inp["txt"], 0.8, inp["ids"], ident, b.H)
    assert v0.shape == (6, 8)
    np.testing.assert_array_equal(v0, v1)
    # the real blocks do change it
    v2 = O.flux_velocity(tok, inp["txt"], 0.8, inp["ids"], m, b.H)
    assert np.abs(v2 - v0).max() > 1e-3


def test_synth_bias_variant_changes_only_biases_and_scales():
    s = synth.BlockShape("bv", 4, 2, 2, 256, 2, 256)
    w0 = synth.single_block_weights(s)
    w1 = synth.single_block_weights(s, bias_std=0.1, norm_scale_std=0.1)
    for k in ("W_mod", "W1", "W2"):
        np.testing.assert_array_equal(w0[k], w1[k])
    for k in ("b_mod", "b1", "b2"):
        b = synth.bf16_bits_to_f64(w1[k])
        assert abs(b.std() - 0.1) < 0.03 and np.count_nonzero(b) > 0.9 * b.size
    for k in ("q_scale", "k_scale"):
        sc = synth.bf16_bits_to_f64(w1[k])
        assert abs(sc.mean() - 1.0) < 0.05 and sc.std() > 0.05
    zm = synth.single_block_weights(s, zero_mod=True, bias_std=0.1)
    assert not synth.bf16_bits_to_f64(zm["b_mod"]).any()  # zero modulation stays the identity


def test_flux_velocity_image_permutation_equivariance():
    """Moving image tokens together with their position ids permutes the
    velocity rows the same way (no mask; RoPE depends on the ids only), for a
    model with real double and single blocks.  This fails if the blocks ever
    see a token next to another token's ids (for example image rows placed
    before the text in the joint sequence while the ids keep text first)."""
    b = synth.BlockShape("vp", 5, 2, 3, 256, 2, 256)
    ls = synth.loop_shape(b, 1, 1, 1, channels=2, txt_in=64)
    m = synth.to_f64(synth.model_weights(ls, bias_std=0.1, norm_scale_std=0.1))
    m = _scale_mod(m, 8.0)
    inp = synth.to_f64(synth.loop_inputs(ls))
    tok = O.patchify(inp["latent"])
    ids = inp["ids"]
    perm = np.array([4, 0, 5, 2, 1, 3])
    ids_p = ids.copy()
    ids_p[b.n_txt:] = ids[b.n_txt:][perm]
    v = O.flux_velocity(tok, inp["txt"], 0.6, ids, m, b.H)
    vp = O.flux_velocity(tok[perm], inp["txt"], 0.6, ids_p, m, b.H)
    np.testing.assert_allclose(vp, v[perm], rtol=1e-10, atol=1e-12)
    # and the ids matter: the same permutation of the tokens alone changes the result
    vq = O.flux_velocity(tok[perm], inp["txt"], 0.6, ids, m, b.H)
    assert np.abs(vq - v[perm]).max() > 1e-4


def _scale_mod(m, k):
    """Every block's adaLN weight times k: larger gates, so that each block's
    branch moves its residual stream visibly."""
    for blk in m["double"]:
        for st in ("txt", "img"):
            blk[st]["W_mod"] = blk[st]["W_mod"] * k
    for blk in m["single"]:
        blk["W_mod"] = blk["W_mod"] * k
    return m
