"""The allocation-free single-block entry point, for callers that may not
allocate device memory (plug-ins inside a framework that owns all device
memory, serving loops that must not call cudaMalloc once running).

It must give the same result as dit_single_block_fwd with a caller-provided
workspace, call after call, although its intermediates live in a fixed array
inside the library that keeps the previous call's contents.  This file is
collected last so that a failure here leaves every other test already run."""
import numpy as np
import pytest

from oracle import dit_oracle as O
from diffusion_transformer_block_flux_b200 import synth
import diffusion_transformer_block_flux_b200 as dit
from helpers import dev_bf16, dev_tree, host_f64, parity

pytestmark = pytest.mark.gpu


def _inputs(seed, biased=False):
    import torch
    s = synth.TINY
    kw = dict(bias_std=synth.TEST_BIAS_STD, norm_scale_std=synth.TEST_NORM_SCALE_STD) if biased else {}
    wb = synth.single_block_weights(s, seed=seed, **kw)
    ab = synth.block_activations(s, seed=seed + 1)
    w = dev_tree(wb)
    x = dev_bf16(ab["x"])
    vec = dev_bf16(ab["vec"]).reshape(1, -1)
    rope = torch.empty((s.S, 64, 2), dtype=torch.float32, device="cuda")
    dit.dit_rope_table(torch.from_numpy(ab["ids"]).cuda(), (8, 28, 28), 10000.0, rope)
    cfg = dit.block_cfg(1, s.S, s.D, s.H, s.M)
    return cfg, w, x, vec, rope, wb, ab


def test_noalloc_matches_workspace_entry_point_twice():
    """Both paths run the same kernels on the same inputs, so the outputs must
    be bit-identical; the second call (other weights, other inputs) finds the
    first call's leftovers in the scratch array.  Each output is also checked
    against the fp64 oracle."""
    import torch
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    s = synth.TINY
    for call, (seed, biased) in enumerate(((0, False), (7, True))):  # two calls in a row, different inputs
        cfg, w, x, vec, rope, wb, ab = _inputs(seed, biased)
        cw = dit.single_weights(w)
        ws = torch.empty(dit.dit_single_block_workspace(cfg), dtype=torch.uint8, device="cuda")
        ref = torch.empty_like(x)
        dit.dit_single_block_fwd(cfg, cw, x, vec, rope, ref, ws)
        out = torch.full_like(x, float("nan"))
        dit.dit_single_block_fwd_noalloc(cfg, cw, x, vec, rope, out)
        torch.cuda.synchronize()
        assert torch.equal(out, ref), f"no-alloc call {call} differs from the workspace call"
        f = synth.to_f64(ab)
        oracle = O.single_block(f["x"], f["vec"], f["ids"], synth.to_f64(wb), s.H)
        parity(host_f64(out), oracle, f"no-alloc call {call} vs oracle")
    st, code = dit.dit_get_device_error()
    assert st == 0, f"device error word {code:#x}"


def test_noalloc_rejects_configs_beyond_its_scratch():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    cfg, w, x, vec, rope, _, _ = _inputs(0)
    big = dit.block_cfg(1, 4608, 3072, 24, 12288)  # needs ~254 MB of intermediates
    with pytest.raises(dit.DitError) as e:
        dit.dit_single_block_fwd_noalloc(big, dit.single_weights(w), x, vec, rope, x)
    assert e.value.code == dit.DIT_ERR_WORKSPACE
