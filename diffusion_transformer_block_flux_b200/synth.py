"""Seeded synthetic inputs for the DiT block workloads.

This module only draws random numbers and lays out shapes and position ids.
It holds none of the block's arithmetic, so both the CUDA path and the CPU
oracle may consume what it produces.

Distributions follow the workload descriptions: linear weights ~ N(0, 0.02),
biases 0, RMSNorm scales 1, tokens and conditioning ~ N(0, 1).  Every tensor
gets its own generator seeded from (seed, crc32(name)), so a tensor's values do
not depend on which other tensors were drawn.  Values are rounded to bf16
(round-to-nearest-even) and returned as raw uint16 bit patterns.
"""
from __future__ import annotations

import zlib
from dataclasses import dataclass

import numpy as np

WEIGHT_STD = 0.02


# --------------------------------------------------------------------------
# bf16 bit patterns
# --------------------------------------------------------------------------


def f32_to_bf16_bits(a) -> np.ndarray:
    """Round float32 values to bf16 (nearest-even); return uint16 bits."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


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


def single_block_weights(shape: BlockShape, seed: int = 0, prefix: str = "single",
                         norm_scale_std: float = 0.0, zero_mod: bool = False) -> dict:
    D, M, d = shape.D, shape.M, shape.d
    w = {
        "W_mod": const_bf16((3 * D, D), 0.0) if zero_mod else _w(seed, f"{prefix}.W_mod", (3 * D, D)),
        "b_mod": const_bf16((3 * D,), 0.0),
        "W1": _w(seed, f"{prefix}.W1", (3 * D + M, D)),
        "b1": const_bf16((3 * D + M,), 0.0),
        "W2": _w(seed, f"{prefix}.W2", (D, D + M)),
        "b2": const_bf16((D,), 0.0),
    }
    for nm in ("q_scale", "k_scale"):
        if norm_scale_std > 0:
            w[nm] = normal_bf16(seed, f"{prefix}.{nm}", (d,), norm_scale_std, 1.0)
        else:
            w[nm] = const_bf16((d,), 1.0)
    return w


def double_block_weights(shape: BlockShape, seed: int = 0, prefix: str = "double",
                         zero_mod: bool = False) -> dict:
    D, M, d = shape.D, shape.M, shape.d
    out = {}
    for s in ("txt", "img"):
        p = f"{prefix}.{s}"
        out[s] = {
            "W_mod": const_bf16((6 * D, D), 0.0) if zero_mod else _w(seed, p + ".W_mod", (6 * D, D)),
            "b_mod": const_bf16((6 * D,), 0.0),
            "W_qkv": _w(seed, p + ".W_qkv", (3 * D, D)),
            "b_qkv": const_bf16((3 * D,), 0.0),
            "q_scale": const_bf16((d,), 1.0),
            "k_scale": const_bf16((d,), 1.0),
            "W_proj": _w(seed, p + ".W_proj", (D, D)),
            "b_proj": const_bf16((D,), 0.0),
            "W_mlp1": _w(seed, p + ".W_mlp1", (M, D)),
            "b_mlp1": const_bf16((M,), 0.0),
            "W_mlp2": _w(seed, p + ".W_mlp2", (D, M)),
            "b_mlp2": const_bf16((D,), 0.0),
        }
    return out


def video_block_weights(shape: VideoShape, seed: int = 0, prefix: str = "video") -> dict:
    D, M = shape.D, shape.M
    names = {
        "W_mod": (6 * D, D), "W_qkv": (3 * D, D), "W_o": (D, D), "W_cq": (D, D),
        "W_ckv": (2 * D, D), "W_co": (D, D), "W_f1": (M, D), "W_f2": (D, M),
    }
    w = {}
    for nm, shp in names.items():
        w[nm] = _w(seed, f"{prefix}.{nm}", shp)
        w["b" + nm[1:]] = const_bf16((shp[0],), 0.0)
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


def model_weights(ls: LoopShape, seed: int = 0) -> dict:
    b = ls.block
    D = b.D
    cin = ls.channels * 4
    m = {
        "W_img_in": _w(seed, "img_in.W", (D, cin)), "b_img_in": const_bf16((D,), 0.0),
        "W_txt_in": _w(seed, "txt_in.W", (D, ls.txt_in)), "b_txt_in": const_bf16((D,), 0.0),
        "W_t1": _w(seed, "time_in.W1", (D, ls.t_dim)), "b_t1": const_bf16((D,), 0.0),
        "W_t2": _w(seed, "time_in.W2", (D, D)), "b_t2": const_bf16((D,), 0.0),
        "W_fmod": _w(seed, "final.W_mod", (2 * D, D)), "b_fmod": const_bf16((2 * D,), 0.0),
        "W_out": _w(seed, "final.W_out", (cin, D)), "b_out": const_bf16((cin,), 0.0),
    }
    m["double"] = [double_block_weights(b, seed, prefix=f"double{i}") for i in range(ls.n_double)]
    m["single"] = [single_block_weights(b, seed, prefix=f"single{i}") for i in range(ls.n_single)]
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
