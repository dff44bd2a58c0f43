"""GPU checks of the whole denoising loop (embedders, double- and single-
stream blocks, final layer, flow-match Euler) through the C ABI: the CUDA
graph replays exactly the eager kernel sequence, and the result matches the
fp64 oracle."""
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


def _scale_modulation(mw, k):
    """Every block's adaLN weight times k (exact in bf16 for a power of two)."""
    sc = lambda a: synth.f32_to_bf16_bits(synth.bf16_bits_to_f32(a) * np.float32(k))
    for blk in mw["double"]:
        for st in ("txt", "img"):
            blk[st]["W_mod"] = sc(blk[st]["W_mod"])
    for blk in mw["single"]:
        blk["W_mod"] = sc(blk["W_mod"])
    return mw


BIAS_NORM = dict(bias_std=synth.TEST_BIAS_STD, norm_scale_std=synth.TEST_NORM_SCALE_STD)


def setup_loop(ls, seed=0, fresh=None, cache_order=1, guidance=None, cfg_steps=-1, mod_scale=1, biased=False):
    """guidance: None = no classifier-free guidance; otherwise the scale, with
    a seeded unconditional text inp["txt_uncond"] of the text's shape.
    mod_scale: multiplies every block's adaLN weight (larger gates give the
    text a visible effect on the image velocity).  biased: the test-only
    weight variant (every bias N(0, 0.1), q/k norm scales N(1, 0.1))."""
    import torch
    b = ls.block
    mw = synth.model_weights(ls, seed=seed, **(BIAS_NORM if biased else {}))
    if mod_scale != 1:
        mw = _scale_modulation(mw, mod_scale)
    inp = synth.loop_inputs(ls, seed=seed + 1)
    mdev = dev_tree(mw)
    model = dit.Model(mdev, D=b.D, H=b.H, M=b.M, channels=ls.channels, txt_dim=ls.txt_in, t_dim=ls.t_dim)
    lat_in = dev_bf16(inp["latent"])
    txt = dev_bf16(inp["txt"])
    unc = None
    if guidance is not None:
        inp["txt_uncond"] = synth.normal_bf16(seed + 2, "txt_uncond", inp["txt"].shape)
        unc = dev_bf16(inp["txt_uncond"])
    ids = torch.from_numpy(inp["ids"]).cuda()
    lat_out = torch.empty(inp["latent"].shape, dtype=torch.float32, device="cuda")
    io = dit.loop_io(b.n_txt, b.grid_h, b.grid_w, ls.steps, lat_in, txt, ids, lat_out, fresh=fresh,
                     cache_order=cache_order, txt_uncond=unc, guidance=1.0 if guidance is None else guidance,
                     cfg_steps=cfg_steps)
    ws = torch.empty(dit.dit_forward_workspace(model, io), dtype=torch.uint8, device="cuda")
    keep = (mdev, lat_in, txt, ids, unc)
    return mw, inp, model, io, ws, lat_out, keep


SMALL = synth.loop_shape(synth.BlockShape("loop_small", 16, 4, 6, 256, 2, 512), 2, 2, 3, channels=16, txt_in=64)


def test_graph_replay_equals_eager_bitwise():
    import torch
    mw, inp, model, io, ws, lat_out, keep = setup_loop(SMALL)
    dit.dit_forward_eager(model, io, ws)
    torch.cuda.synchronize()
    eager = lat_out.clone()
    lat_out.zero_()
    g = dit.Graph(model, io, ws)
    assert g.nodes() > 4 * SMALL.steps
    g.launch()
    torch.cuda.synchronize()
    assert torch.equal(lat_out, eager)
    lat_out.zero_()
    g.launch()  # replay again: same bits
    torch.cuda.synchronize()
    assert torch.equal(lat_out, eager)
    g.destroy()
    st, code = dit.dit_get_device_error()
    assert st == 0, f"device error word {code:#x}"


@pytest.mark.parametrize("biased", [False, True])
def test_loop_matches_oracle_small(biased):
    import torch
    mw, inp, model, io, ws, lat_out, keep = setup_loop(SMALL, biased=biased)
    g = dit.Graph(model, io, ws)
    g.launch()
    torch.cuda.synchronize()
    got = lat_out.cpu().double().numpy()
    f = synth.to_f64(inp)
    ref = O.euler_sample(f["latent"], f["txt"], f["ids"], synth.to_f64(mw), SMALL.block.H, SMALL.steps)
    parity(got, ref, "final latent")
    # the displacement x_T - x_0 is the integrated velocity; check it alone too
    parity(got - f["latent"], ref - f["latent"], "integrated velocity")
    g.destroy()


@pytest.mark.parametrize("biased", [False, True])
def test_full_depth_velocity_at_tiny_dims(biased):
    """19 double + 38 single blocks at dim 384 (S = 64 + 192): one Euler step
    from t=1 to 0 moves the latent by exactly -v(x0, 1), the model forward."""
    import torch
    ls = synth.loop_shape(synth.TINY, 19, 38, 1, channels=16, txt_in=4096)
    mw, inp, model, io, ws, lat_out, keep = setup_loop(ls, biased=biased)
    dit.dit_forward_eager(model, io, ws)
    torch.cuda.synchronize()
    got = lat_out.cpu().double().numpy()
    f = synth.to_f64(inp)
    ref = O.euler_sample(f["latent"], f["txt"], f["ids"], synth.to_f64(mw), ls.block.H, 1)
    # Derived tolerance for a chain of L = 57 blocks: each block stores its
    # residual output in bf16 (relative RMS rounding error about 2^-8/sqrt(3),
    # about 2.3e-3, plus its internal roundings; about 1.6e-3 measured per block).
    # Independent per-block errors add in quadrature, so the chain is allowed
    # 2.5e-3 * sqrt(57), about 1.9e-2, on rel L2; max abs scales the same way
    # (6e-2 RMS).
    parity(got - f["latent"], ref - f["latent"], "full-depth velocity", rel_l2=2e-2, max_abs_frac=6e-2)
    parity(got, ref, "full-depth latent", max_abs_frac=6e-2)


CACHED = synth.loop_shape(synth.BlockShape("loop_small", 16, 4, 6, 256, 2, 512), 2, 2, 6, channels=16, txt_in=64)


def test_step_cache_all_fresh_is_bitwise_the_plain_loop():
    import torch
    _, _, model, io, ws, lat_out, keep = setup_loop(CACHED)
    dit.dit_forward_eager(model, io, ws)
    torch.cuda.synchronize()
    plain = lat_out.clone()
    _, _, model2, io2, ws2, lat_out2, keep2 = setup_loop(CACHED, fresh=[1] * CACHED.steps)
    dit.dit_forward_eager(model2, io2, ws2)
    torch.cuda.synchronize()
    assert torch.equal(plain, lat_out2)


@pytest.mark.parametrize("order,biased", [(0, False), (1, False), (1, True)])
def test_step_cache_matches_oracle_and_graph_equals_eager(order, biased):
    """Model-level step cache: steps 2, 4, 5 predicted from kept velocities."""
    import torch
    fresh = [1, 1, 0, 1, 0, 0]
    mw, inp, model, io, ws, lat_out, keep = setup_loop(CACHED, fresh=fresh, cache_order=order, biased=biased)
    dit.dit_forward_eager(model, io, ws)
    torch.cuda.synchronize()
    eager = lat_out.clone()
    g = dit.Graph(model, io, ws)
    lat_out.zero_()
    g.launch()
    torch.cuda.synchronize()
    assert torch.equal(lat_out, eager)
    g.destroy()
    f = synth.to_f64(inp)
    ref = O.euler_sample(f["latent"], f["txt"], f["ids"], synth.to_f64(mw), CACHED.block.H, CACHED.steps,
                         fresh=fresh, cache_order=order)
    got = eager.cpu().double().numpy()
    parity(got, ref, f"cached loop (order {order})")
    parity(got - f["latent"], ref - f["latent"], f"cached loop displacement (order {order})")
    st, code = dit.dit_get_device_error()
    assert st == 0, f"device error word {code:#x}"


@pytest.mark.parametrize("cfg_steps,fresh,biased", [(-1, None, False), (4, None, False),
                                                    (-1, [1, 1, 0, 1, 0, 0], False), (4, None, True)])
def test_guided_loop_matches_oracle_and_graph_equals_eager(cfg_steps, fresh, biased):
    """Classifier-free guidance (scale 1.5): every step, only the first four
    steps, and with the step cache predicting from guided velocities.  The
    adaLN weights are scaled by 32 so that the text moves the image velocity
    by several percent; the test first checks that the guided and unguided
    references differ by more than the tolerance, so it can tell them apart."""
    import torch
    g = 1.5
    mw, inp, model, io, ws, lat_out, keep = setup_loop(CACHED, guidance=g, cfg_steps=cfg_steps, fresh=fresh,
                                                       mod_scale=32, biased=biased)
    dit.dit_forward_eager(model, io, ws)
    torch.cuda.synchronize()
    eager = lat_out.clone()
    graph = dit.Graph(model, io, ws)
    lat_out.zero_()
    graph.launch()
    torch.cuda.synchronize()
    assert torch.equal(lat_out, eager)
    graph.destroy()
    f = synth.to_f64(inp)
    ref = O.euler_sample(f["latent"], f["txt"], f["ids"], synth.to_f64(mw), CACHED.block.H, CACHED.steps,
                         fresh=fresh, txt_uncond=f["txt_uncond"], guidance=g,
                         cfg_steps=None if cfg_steps < 0 else cfg_steps)
    unguided = O.euler_sample(f["latent"], f["txt"], f["ids"], synth.to_f64(mw), CACHED.block.H, CACHED.steps,
                              fresh=fresh)
    d = ref - f["latent"]
    assert np.linalg.norm(unguided - ref) / np.linalg.norm(d) > 1.4e-2  # guidance is visible
    got = eager.cpu().double().numpy()
    parity(got, ref, f"guided loop (cfg_steps {cfg_steps})")
    parity(got - f["latent"], ref - f["latent"], f"guided loop displacement (cfg_steps {cfg_steps})")
    st, code = dit.dit_get_device_error()
    assert st == 0, f"device error word {code:#x}"


class _LazyF64Blocks:
    """A model's block list converted to float64 one block at a time, as the
    oracle walks it (the float64 copy of every block at once would not fit)."""

    def __init__(self, blocks):
        self.blocks = blocks

    def __len__(self):
        return len(self.blocks)

    def __iter__(self):
        for blk in self.blocks:
            yield synth.to_f64(blk)


def test_full_dim_loop_velocity_matches_oracle():
    """The loop at the Flux model's width and depth: dim 3072, 24 heads,
    19 double + 38 single blocks, on a short sequence (64 text + 8 x 8 image
    tokens, MLP hidden 256 to keep the weights at 12 GB) with the biased weight
    variant, one Euler step captured as a graph.  Every block's modulation of
    the step comes from one batched pass over all 77 modulation matrices
    (K = 3072), the path the full-size loop runs."""
    import torch
    b = synth.BlockShape("loop_dim3072", 64, 8, 8, 3072, 24, 256)
    ls = synth.loop_shape(b, 19, 38, 1, channels=16, txt_in=4096)
    mw, inp, model, io, ws, lat_out, keep = setup_loop(ls, biased=True)
    g = dit.Graph(model, io, ws)
    g.launch()
    torch.cuda.synchronize()
    g.destroy()
    st, code = dit.dit_get_device_error()
    assert st == 0, f"device error word {code:#x}"
    got = lat_out.cpu().double().numpy()
    del model, io, ws, keep
    torch.cuda.empty_cache()
    f = synth.to_f64(inp)
    m64 = {k: synth.to_f64(v) for k, v in mw.items() if k not in ("double", "single")}
    m64["double"] = _LazyF64Blocks(mw["double"])
    m64["single"] = _LazyF64Blocks(mw["single"])
    ref = O.euler_sample(f["latent"], f["txt"], f["ids"], m64, b.H, 1)
    # the 57-block chain tolerance of test_full_depth_velocity_at_tiny_dims;
    # one step from t = 1 to 0 moves the latent by -v exactly, so the latent's
    # error is the velocity's, whose max is bounded by the chain's 6e-2 RMS(v)
    parity(got - f["latent"], ref - f["latent"], "dim-3072 full-depth velocity", rel_l2=2e-2, max_abs_frac=6e-2)
    parity(got, ref, "dim-3072 full-depth latent", max_abs_frac=6e-2)
