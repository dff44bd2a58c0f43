"""Test helpers: host<->device transfer of bf16 bit patterns and the parity
check used by every GPU test.

Tolerance (bf16 outputs, fp32 accumulation on the GPU vs the fp64 oracle):
relative L2 error <= 1e-2 and max |error| <= 3e-2 * RMS(reference).
"""
import numpy as np

from diffusion_transformer_block_flux_b200 import synth

REL_L2 = 1e-2
MAX_ABS_FRAC = 3e-2


def dev_bf16(bits, device="cuda"):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def dev_tree(tree, device="cuda"):
    if isinstance(tree, dict):
        return {k: dev_tree(v, device) for k, v in tree.items()}
    if isinstance(tree, list):
        return [dev_tree(v, device) for v in tree]
    if isinstance(tree, np.ndarray) and tree.dtype == np.uint16:
        return dev_bf16(tree, device)
    if isinstance(tree, np.ndarray):
        import torch
        return torch.from_numpy(np.ascontiguousarray(tree)).to(device)
    return tree


def host_f64(t):
    import torch
    if t.dtype == torch.bfloat16:
        return synth.bf16_bits_to_f64(t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16))
    return t.detach().double().cpu().numpy()


def parity(got, ref, what="", rel_l2=REL_L2, max_abs_frac=MAX_ABS_FRAC, resid_roundings=0):
    """resid_roundings: bf16 roundings the residual stream passes through
    inside the checked computation beyond the output's own (a double-stream
    block stores x after its attention branch before adding the MLP branch).
    Each adds up to half an ulp, 2^-9 relative, at the element's own
    magnitude, so the max-abs bound grows by resid_roundings * 2^-9 * max|ref|
    (independent of the RMS the stated bound scales with)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = got - ref
    nref = np.linalg.norm(ref)
    rl2 = np.linalg.norm(err) / max(nref, 1e-300)
    rms = nref / np.sqrt(ref.size)
    mab = np.abs(err).max()
    bound = max_abs_frac * rms + resid_roundings * 2.0 ** -9 * np.abs(ref).max()
    assert rl2 <= rel_l2, f"{what}: rel L2 {rl2:.3e} > {rel_l2}"
    assert mab <= bound, (f"{what}: max abs {mab:.3e} > {max_abs_frac} * RMS {rms:.3e}"
                          + (f" + {resid_roundings} * 2^-9 * max|ref|" if resid_roundings else ""))
    return rl2, mab / rms
