"""Seeded synthetic inputs for the DiT block workloads.

This module only draws random numbers and lays out shapes and position ids.
It holds none of the block's arithmetic, so both the CUDA path and the CPU
oracle may consume what it produces.

Distributions follow the workload descriptions: linear weights ~ N(0, 0.02),
biases 0, RMSNorm scales 1, tokens and conditioning ~ N(0, 1).  A test-only
variant (bias_std > 0, norm_scale_std > 0) draws every bias from N(0, bias_std)
and the q/k RMSNorm scales from N(1, norm_scale_std), so that the bias and
scale wiring of every kernel and block is exercised too.  Every tensor
gets its own generator seeded from (seed, crc32(name)), so a tensor's values do
not depend on which other tensors were drawn.  Values are rounded to bf16
(round-to-nearest-even) and returned as raw uint16 bit patterns.
"""
from __future__ import annotations

import os
import zlib
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass

import numpy as np

WEIGHT_STD = 0.02
# the test-only variant: nonzero biases and non-unit q/k norm scales
TEST_BIAS_STD = 0.1
TEST_NORM_SCALE_STD = 0.1


# --------------------------------------------------------------------------
# bf16 bit patterns
# --------------------------------------------------------------------------


def f32_to_bf16_bits(a) -> np.ndarray:
    """Round float32 values to bf16 (nearest-even); return uint16 bits.
    In 32-bit integer arithmetic: for every finite value (and +-inf) the sum
    below stays under 2^32; NaNs map to the canonical quiet NaN."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32)
    r = u + np.uint32(0x7FFF)
    r += (u >> np.uint32(16)) & np.uint32(1)
    r >>= np.uint32(16)
    out = r.astype(np.uint16)
    nan = np.isnan(a)
    if nan.any():
        out[nan] = 0x7FC0
    return out


def bf16_bits_to_f64(b) -> np.ndarray:
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def bf16_bits_to_f32(b) -> np.ndarray:
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def _rng(seed: int, name: str) -> np.random.Generator:
    return np.random.default_rng([int(seed) & 0xFFFFFFFF, zlib.crc32(name.encode())])


def normal_bf16(seed: int, name: str, shape, std: float = 1.0, mean: float = 0.0) -> np.ndarray:
    g = _rng(seed, name)
    a = g.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    if mean != 0.0:
        a += np.float32(mean)
    return f32_to_bf16_bits(a)


def const_bf16(shape, value: float) -> np.ndarray:
    return f32_to_bf16_bits(np.full(shape, value, dtype=np.float32))


# --------------------------------------------------------------------------
# Position ids (structure of the token sequence, not arithmetic)
# --------------------------------------------------------------------------


def flux_ids(n_txt: int, grid_h: int, grid_w: int) -> np.ndarray:
    """[n_txt + gh*gw, 3] int32: text tokens at (0,0,0) first, then image
    tokens at (0, h, w) in row-major patch order."""
    ids = np.zeros((n_txt + grid_h * grid_w, 3), dtype=np.int32)
    hh, ww = np.meshgrid(np.arange(grid_h), np.arange(grid_w), indexing="ij")
    ids[n_txt:, 1] = hh.reshape(-1)
    ids[n_txt:, 2] = ww.reshape(-1)
    return ids


def video_ids(frames: int, grid_h: int, grid_w: int) -> np.ndarray:
    """[f*gh*gw, 3] int32 (t, h, w) in row-major order."""
    t, h, w = np.meshgrid(np.arange(frames), np.arange(grid_h), np.arange(grid_w),
                          indexing="ij")
    return np.stack([t.reshape(-1), h.reshape(-1), w.reshape(-1)], axis=1).astype(np.int32)


# --------------------------------------------------------------------------
# Workloads
# --------------------------------------------------------------------------


@dataclass(frozen=True)
class BlockShape:
    name: str
    n_txt: int
    grid_h: int
    grid_w: int
    D: int
    H: int
    M: int
    d: int = 128

    @property
    def S(self) -> int:
        return self.n_txt + self.grid_h * self.grid_w


# Tiny single-stream block: 64 text + 12x16 image tokens, dim 384, 3 heads.
TINY = BlockShape("tiny_single_S256_D384", 64, 12, 16, 384, 3, 1536)
# Flux.1-dev single/double-stream block at 1024^2: 512 text + 64x64 image tokens.
FLUX = BlockShape("flux_single_S4608_D3072", 512, 64, 64, 3072, 24, 12288)
FLUX_DOUBLE = BlockShape("flux_double_T512_I4096_D3072", 512, 64, 64, 3072, 24, 12288)


@dataclass(frozen=True)
class VideoShape:
    name: str
    frames: int
    grid_h: int
    grid_w: int
    D: int
    H: int
    M: int
    n_ctx: int
    ctx_in: int = 4096
    d: int = 128

    @property
    def S(self) -> int:
        return self.frames * self.grid_h * self.grid_w


# Wan2.1-1.3B-shaped block: 21 latent frames x 30 x 45 patches, dim 1536.
VIDEO = VideoShape("video_block_S28350_D1536", 21, 30, 45, 1536, 12, 8960, 512)


def _w(seed, name, shape, std=WEIGHT_STD):
    return normal_bf16(seed, name, shape, std)


def _b(seed, name, n, bias_std):
    """A bias: zero in the workload recipe, N(0, bias_std) in the test variant."""
    return normal_bf16(seed, name, (n,), bias_std) if bias_std > 0 else const_bf16((n,), 0.0)


def _s(seed, name, d, norm_scale_std):
    """An RMSNorm scale: one in the workload recipe, N(1, std) in the test variant."""
    return normal_bf16(seed, name, (d,), norm_scale_std, 1.0) if norm_scale_std > 0 else const_bf16((d,), 1.0)


def single_block_weights(shape: BlockShape, seed: int = 0, prefix: str = "single",
                         norm_scale_std: float = 0.0, zero_mod: bool = False, bias_std: float = 0.0) -> dict:
    """zero_mod: W_mod and b_mod zero (shift = scale = gate = 0: the block is the identity)."""
    D, M, d = shape.D, shape.M, shape.d
    w = {
        "W_mod": const_bf16((3 * D, D), 0.0) if zero_mod else _w(seed, f"{prefix}.W_mod", (3 * D, D)),
        "b_mod": _b(seed, f"{prefix}.b_mod", 3 * D, 0.0 if zero_mod else bias_std),
        "W1": _w(seed, f"{prefix}.W1", (3 * D + M, D)),
        "b1": _b(seed, f"{prefix}.b1", 3 * D + M, bias_std),
        "W2": _w(seed, f"{prefix}.W2", (D, D + M)),
        "b2": _b(seed, f"{prefix}.b2", D, bias_std),
    }
    for nm in ("q_scale", "k_scale"):
        w[nm] = _s(seed, f"{prefix}.{nm}", d, norm_scale_std)
    return w


def double_block_weights(shape: BlockShape, seed: int = 0, prefix: str = "double",
                         zero_mod: bool = False, bias_std: float = 0.0, norm_scale_std: float = 0.0) -> dict:
    D, M, d = shape.D, shape.M, shape.d
    out = {}
    for s in ("txt", "img"):
        p = f"{prefix}.{s}"
        out[s] = {
            "W_mod": const_bf16((6 * D, D), 0.0) if zero_mod else _w(seed, p + ".W_mod", (6 * D, D)),
            "b_mod": _b(seed, p + ".b_mod", 6 * D, 0.0 if zero_mod else bias_std),
            "W_qkv": _w(seed, p + ".W_qkv", (3 * D, D)),
            "b_qkv": _b(seed, p + ".b_qkv", 3 * D, bias_std),
            "q_scale": _s(seed, p + ".q_scale", d, norm_scale_std),
            "k_scale": _s(seed, p + ".k_scale", d, norm_scale_std),
            "W_proj": _w(seed, p + ".W_proj", (D, D)),
            "b_proj": _b(seed, p + ".b_proj", D, bias_std),
            "W_mlp1": _w(seed, p + ".W_mlp1", (M, D)),
            "b_mlp1": _b(seed, p + ".b_mlp1", M, bias_std),
            "W_mlp2": _w(seed, p + ".W_mlp2", (D, M)),
            "b_mlp2": _b(seed, p + ".b_mlp2", D, bias_std),
        }
    return out


def video_block_weights(shape: VideoShape, seed: int = 0, prefix: str = "video", bias_std: float = 0.0) -> dict:
    D, M = shape.D, shape.M
    names = {
        "W_mod": (6 * D, D), "W_qkv": (3 * D, D), "W_o": (D, D), "W_cq": (D, D),
        "W_ckv": (2 * D, D), "W_co": (D, D), "W_f1": (M, D), "W_f2": (D, M),
    }
    w = {}
    for nm, shp in names.items():
        w[nm] = _w(seed, f"{prefix}.{nm}", shp)
        w["b" + nm[1:]] = _b(seed, f"{prefix}.b{nm[1:]}", shp[0], bias_std)
    return w


def block_activations(shape: BlockShape, seed: int = 1) -> dict:
    return {
        "x": normal_bf16(seed, "x", (shape.S, shape.D)),
        "vec": normal_bf16(seed, "vec", (shape.D,)),
        "ids": flux_ids(shape.n_txt, shape.grid_h, shape.grid_w),
    }


def double_block_activations(shape: BlockShape, seed: int = 1) -> dict:
    return {
        "img": normal_bf16(seed, "img", (shape.grid_h * shape.grid_w, shape.D)),
        "txt": normal_bf16(seed, "txt", (shape.n_txt, shape.D)),
        "vec": normal_bf16(seed, "vec", (shape.D,)),
        "ids": flux_ids(shape.n_txt, shape.grid_h, shape.grid_w),
    }


def video_activations(shape: VideoShape, seed: int = 1) -> dict:
    return {
        "x": normal_bf16(seed, "x", (shape.S, shape.D)),
        "ctx": normal_bf16(seed, "ctx", (shape.n_ctx, shape.D)),
        "vec": normal_bf16(seed, "vec", (shape.D,)),
        "ids": video_ids(shape.frames, shape.grid_h, shape.grid_w),
    }


@dataclass(frozen=True)
class LoopShape:
    name: str
    block: BlockShape
    channels: int
    n_double: int
    n_single: int
    steps: int
    txt_in: int = 4096
    t_dim: int = 256


# Flux.1-dev loop at 1024^2: 16x128x128 latent, 19 double + 38 single, 50 steps.
FLUX_LOOP = LoopShape("flux_loop_1024px_57blocks_50steps", FLUX, 16, 19, 38, 50)


def loop_shape(block: BlockShape, n_double: int, n_single: int, steps: int,
               channels: int = 16, txt_in: int = 4096) -> LoopShape:
    return LoopShape(f"loop_{block.name}_{n_double}d{n_single}s_{steps}steps", block,
                     channels, n_double, n_single, steps, txt_in)


def model_weights(ls: LoopShape, seed: int = 0, bias_std: float = 0.0, norm_scale_std: float = 0.0) -> dict:
    b = ls.block
    D = b.D
    cin = ls.channels * 4
    m = {
        "W_img_in": _w(seed, "img_in.W", (D, cin)), "b_img_in": _b(seed, "img_in.b", D, bias_std),
        "W_txt_in": _w(seed, "txt_in.W", (D, ls.txt_in)), "b_txt_in": _b(seed, "txt_in.b", D, bias_std),
        "W_t1": _w(seed, "time_in.W1", (D, ls.t_dim)), "b_t1": _b(seed, "time_in.b1", D, bias_std),
        "W_t2": _w(seed, "time_in.W2", (D, D)), "b_t2": _b(seed, "time_in.b2", D, bias_std),
        "W_fmod": _w(seed, "final.W_mod", (2 * D, D)), "b_fmod": _b(seed, "final.b_mod", 2 * D, bias_std),
        "W_out": _w(seed, "final.W_out", (cin, D)), "b_out": _b(seed, "final.b_out", cin, bias_std),
    }
    # every tensor has its own stream, so the blocks can be drawn concurrently
    # (numpy releases the GIL while filling and converting large arrays)
    with ThreadPoolExecutor(max(1, min(16, os.cpu_count() or 1))) as ex:
        dbl = ex.map(lambda i: double_block_weights(b, seed, prefix=f"double{i}", bias_std=bias_std,
                                                    norm_scale_std=norm_scale_std), range(ls.n_double))
        sgl = ex.map(lambda i: single_block_weights(b, seed, prefix=f"single{i}", bias_std=bias_std,
                                                    norm_scale_std=norm_scale_std), range(ls.n_single))
        m["double"], m["single"] = list(dbl), list(sgl)
    return m


def loop_inputs(ls: LoopShape, seed: int = 1) -> dict:
    b = ls.block
    return {
        "latent": normal_bf16(seed, "latent", (ls.channels, 2 * b.grid_h, 2 * b.grid_w)),
        "txt": normal_bf16(seed, "txt_raw", (b.n_txt, ls.txt_in)),
        "ids": flux_ids(b.n_txt, b.grid_h, b.grid_w),
    }


def to_f64(tree):
    """Map every uint16 bf16 array in a (nested) dict/list to float64."""
    if isinstance(tree, dict):
        return {k: to_f64(v) for k, v in tree.items()}
    if isinstance(tree, list):
        return [to_f64(v) for v in tree]
    if isinstance(tree, np.ndarray) and tree.dtype == np.uint16:
        return bf16_bits_to_f64(tree)
    return tree
