"""B200-native (sm_100a) Flux-style DiT block forward.

The compute lives in libdit.so (hand-written CUDA kernels behind the C ABI in
include/dit.h).  This package is a thin ctypes binding whose functions carry
the C names; it only marshals arguments (pointers, sizes, the current CUDA
stream) and raises DitError on a non-zero status.  There is no fallback: if
libdit.so is missing or fails to load, every call raises.
"""
from __future__ import annotations

import ctypes
import os
import re

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
ROOT_DIR = os.path.dirname(PKG_DIR)
LIB_PATH = os.path.join(PKG_DIR, "libdit.so")
HEADER_PATH = os.path.join(ROOT_DIR, "include", "dit.h")

c_bf16_p = ctypes.c_void_p
c_void_p = ctypes.c_void_p
i32, i64, f32, f64 = ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_double
size_t = ctypes.c_size_t

STATUS = {
    0: "DIT_OK", 1: "DIT_ERR_INVALID_ARG", 2: "DIT_ERR_SHAPE", 3: "DIT_ERR_ALIGNMENT",
    4: "DIT_ERR_UNSUPPORTED", 5: "DIT_ERR_CUDA", 6: "DIT_ERR_NOT_CAPTURABLE",
    7: "DIT_ERR_TIMEOUT", 8: "DIT_ERR_WORKSPACE",
}
DIT_OK, DIT_ERR_INVALID_ARG, DIT_ERR_SHAPE, DIT_ERR_ALIGNMENT = 0, 1, 2, 3
DIT_ERR_UNSUPPORTED, DIT_ERR_CUDA, DIT_ERR_NOT_CAPTURABLE, DIT_ERR_TIMEOUT, DIT_ERR_WORKSPACE = 4, 5, 6, 7, 8
DIT_EPI_NONE, DIT_EPI_BIAS, DIT_EPI_BIAS_GELU_COLS, DIT_EPI_BIAS_GATED_RESIDUAL = 0, 1, 2, 3
DIT_VEC_SILU_IN, DIT_VEC_OUT_BF16 = 1, 2


class DitError(RuntimeError):
    def __init__(self, fn: str, code: int, detail: str = ""):
        super().__init__(f"{fn} returned {STATUS.get(code, code)}" + (f" ({detail})" if detail else ""))
        self.code = code


# ----------------------------------------------------------------------------
# C structs (field order and types mirror include/dit.h)
# ----------------------------------------------------------------------------


class dit_gemm_args(ctypes.Structure):
    _fields_ = [
        ("A", c_void_p), ("lda", i64), ("W", c_void_p), ("ldw", i64), ("bias", c_void_p),
        ("C", c_void_p), ("ldc", i64), ("C2", c_void_p), ("ldc2", i64), ("split_col", i32),
        ("M", i32), ("N", i32), ("K", i32), ("epi", i32), ("gelu_col_begin", i32),
        ("gate", c_void_p), ("gate_stride", i64), ("resid", c_void_p), ("ldr", i64),
        ("rows_per_batch", i32), ("qk_cols", i32), ("qk_norm", i32), ("qk_eps", f32),
        ("q_scale", c_void_p), ("k_scale", c_void_p), ("rope", c_void_p), ("rope_rows", i32),
    ]


class dit_block_cfg(ctypes.Structure):
    _fields_ = [("B", i32), ("S", i32), ("n_txt", i32), ("D", i32), ("H", i32),
                ("head_dim", i32), ("M", i32), ("eps", f32)]


class dit_single_weights(ctypes.Structure):
    _fields_ = [(n, c_void_p) for n in ("W_mod", "b_mod", "W1", "b1", "q_scale", "k_scale", "W2", "b2")]


STREAM_FIELDS = ("W_mod", "b_mod", "W_qkv", "b_qkv", "q_scale", "k_scale", "W_proj", "b_proj",
                 "W_mlp1", "b_mlp1", "W_mlp2", "b_mlp2")


class dit_stream_weights(ctypes.Structure):
    _fields_ = [(n, c_void_p) for n in STREAM_FIELDS]


class dit_double_weights(ctypes.Structure):
    _fields_ = [("txt", dit_stream_weights), ("img", dit_stream_weights)]


VIDEO_FIELDS = ("W_mod", "b_mod", "W_qkv", "b_qkv", "W_o", "b_o", "W_cq", "b_cq", "W_ckv", "b_ckv",
                "W_co", "b_co", "W_f1", "b_f1", "W_f2", "b_f2")


class dit_video_weights(ctypes.Structure):
    _fields_ = [(n, c_void_p) for n in VIDEO_FIELDS]


class dit_model(ctypes.Structure):
    _fields_ = [
        ("D", i32), ("H", i32), ("head_dim", i32), ("M", i32), ("channels", i32), ("txt_dim", i32),
        ("t_dim", i32), ("n_double", i32), ("n_single", i32),
        ("double_blocks", ctypes.POINTER(dit_double_weights)),
        ("single_blocks", ctypes.POINTER(dit_single_weights)),
    ] + [(n, c_void_p) for n in ("W_img_in", "b_img_in", "W_txt_in", "b_txt_in", "W_t1", "b_t1",
                                  "W_t2", "b_t2", "W_fmod", "b_fmod", "W_out", "b_out")] + [("eps", f32)]


class dit_loop_io(ctypes.Structure):
    _fields_ = [("n_txt", i32), ("grid_h", i32), ("grid_w", i32), ("steps", i32),
                ("latent_in", c_void_p), ("txt", c_void_p), ("ids", c_void_p), ("latent_out", c_void_p),
                ("fresh", ctypes.POINTER(ctypes.c_uint8)), ("cache_order", i32),
                ("txt_uncond", c_void_p), ("guidance", f32), ("cfg_steps", i32)]


# ----------------------------------------------------------------------------
# Library loading
# ----------------------------------------------------------------------------

_SIGS = {
    "dit_status_string": (ctypes.c_char_p, [i32]),
    "dit_version": (i32, []),
    "dit_abi_struct_size": (size_t, [i32]),
    "dit_step_cache_plan": (i32, [i32, ctypes.POINTER(ctypes.c_uint8), i32, ctypes.POINTER(i32),
                                  ctypes.POINTER(i32), ctypes.POINTER(i32), ctypes.POINTER(f32),
                                  ctypes.POINTER(f32)]),
    "dit_last_cuda_error": (ctypes.c_char_p, []),
    "dit_get_device_error": (i32, [c_void_p, ctypes.POINTER(ctypes.c_uint32)]),
    "dit_clear_device_error": (i32, [c_void_p]),
    "dit_set_wait_limit_ns": (i32, [ctypes.c_uint64]),
    "dit_selftest_wait_timeout": (i32, [ctypes.c_uint64, c_void_p]),
    "dit_rope_table": (i32, [c_void_p, i32, i32, ctypes.POINTER(i32), f64, c_void_p, c_void_p]),
    "dit_adaln_modulation": (i32, [c_void_p, i64, c_void_p, i64, c_void_p, c_void_p, i64, i32, i32, i32,
                                   c_void_p]),
    "dit_vec_linear": (i32, [c_void_p, i64, c_void_p, i64, c_void_p, c_void_p, i64, i32, i32, i32, i32,
                             c_void_p]),
    "dit_modulate_norm": (i32, [c_void_p, i64, c_void_p, c_void_p, i64, c_void_p, i64, i32, i32, i32, f32,
                                c_void_p]),
    "dit_qk_norm_rope": (i32, [c_void_p, c_void_p, i64, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                               i64, i32, i32, i32, i32, f32, c_void_p]),
    "dit_attention": (i32, [c_void_p, c_void_p, c_void_p, i64, i64, i64, c_void_p, i64, c_void_p, i32, i32,
                            i32, i32, i32, f32, c_void_p]),
    "dit_attention_accumulate": (i32, [c_void_p, c_void_p, c_void_p, i64, i64, i64, c_void_p, i64, c_void_p, i32,
                                       i32, i32, i32, i32, f32, c_void_p]),
    "dit_set_weight_l2_persist": (i32, [size_t]),
    "dit_attention_split": (i32, [c_void_p, c_void_p, c_void_p, i64, i64, i64, c_void_p, i64, c_void_p, i32, i32,
                                  i32, i32, i32, f32, i32, i32, c_void_p, size_t, c_void_p]),
    "dit_attention_split_workspace": (size_t, [i32, i32, i32, i32]),
    "dit_gemm_epilogue": (i32, [ctypes.POINTER(dit_gemm_args), c_void_p]),
    "dit_gemm_epilogue_grouped": (i32, [ctypes.POINTER(dit_gemm_args), ctypes.POINTER(dit_gemm_args), c_void_p]),
    "dit_selftest_exp2_poly": (i32, [c_void_p, c_void_p, i64, c_void_p]),
    "dit_attention_merge": (i32, [i32, ctypes.POINTER(c_void_p), ctypes.POINTER(c_void_p), i64, c_void_p, c_void_p,
                                  i64, i32, i32, i32, c_void_p]),
    "dit_single_block_workspace": (size_t, [ctypes.POINTER(dit_block_cfg)]),
    "dit_double_block_workspace": (size_t, [ctypes.POINTER(dit_block_cfg)]),
    "dit_video_block_workspace": (size_t, [ctypes.POINTER(dit_block_cfg), i32]),
    "dit_single_block_fwd": (i32, [ctypes.POINTER(dit_block_cfg), ctypes.POINTER(dit_single_weights),
                                   c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, size_t, c_void_p]),
    "dit_single_block_fwd_profiled": (i32, [ctypes.POINTER(dit_block_cfg), ctypes.POINTER(dit_single_weights),
                                            c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, size_t,
                                            ctypes.POINTER(c_void_p), i32, c_void_p]),
    "dit_single_block_fwd_noalloc": (i32, [ctypes.POINTER(dit_block_cfg), ctypes.POINTER(dit_single_weights),
                                           c_void_p, c_void_p, c_void_p, c_void_p, c_void_p]),
    "dit_single_block_host_workspace": (size_t, [ctypes.POINTER(dit_block_cfg)]),
    "dit_single_block_fwd_host": (i32, [ctypes.POINTER(dit_block_cfg), ctypes.POINTER(dit_single_weights), i32,
                                        ctypes.POINTER(c_void_p), ctypes.POINTER(c_void_p), ctypes.POINTER(c_void_p),
                                        c_void_p, c_void_p, size_t, c_void_p]),
    "dit_double_block_fwd": (i32, [ctypes.POINTER(dit_block_cfg), ctypes.POINTER(dit_double_weights),
                                   c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                   size_t, c_void_p]),
    "dit_video_block_fwd": (i32, [ctypes.POINTER(dit_block_cfg), ctypes.POINTER(dit_video_weights),
                                  c_void_p, c_void_p, i32, c_void_p, c_void_p, c_void_p, c_void_p, size_t,
                                  c_void_p]),
    "dit_forward_workspace": (size_t, [ctypes.POINTER(dit_model), ctypes.POINTER(dit_loop_io)]),
    "dit_forward_eager": (i32, [ctypes.POINTER(dit_model), ctypes.POINTER(dit_loop_io), c_void_p, size_t,
                                c_void_p]),
    "dit_forward_graph_create": (i32, [ctypes.POINTER(dit_model), ctypes.POINTER(dit_loop_io), c_void_p,
                                       size_t, ctypes.POINTER(c_void_p)]),
    "dit_forward_graph_launch": (i32, [c_void_p, c_void_p]),
    "dit_forward_graph_nodes": (i32, [c_void_p, ctypes.POINTER(size_t)]),
    "dit_forward_graph_destroy": (i32, [c_void_p]),
}

_lib = None


def lib() -> ctypes.CDLL:
    """Load libdit.so (built in-tree by build.py).  Raises if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m diffusion_transformer_block_flux_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def header_functions() -> list[str]:
    """Names of every function declared in include/dit.h."""
    with open(HEADER_PATH) as f:
        txt = f.read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(dit_[a-z0-9_]+)\s*\(", txt)))


def _check(name: str, code: int):
    if code != 0:
        detail = lib().dit_last_cuda_error().decode() if code == DIT_ERR_CUDA else ""
        raise DitError(name, code, detail)


def _call(name: str, *args):
    _check(name, getattr(lib(), name)(*args))


def _stream(stream) -> int:
    if stream is not None:
        return int(stream)
    import torch
    return torch.cuda.current_stream().cuda_stream


def _ptr(t) -> int | None:
    if t is None:
        return None
    return t.data_ptr()


# ----------------------------------------------------------------------------
# Wrappers named after the C entry points (torch tensors in, no compute here)
# ----------------------------------------------------------------------------


def dit_status_string(code: int) -> str:
    return lib().dit_status_string(code).decode()


def dit_version() -> int:
    return lib().dit_version()


def dit_last_cuda_error() -> str:
    return lib().dit_last_cuda_error().decode()


def dit_get_device_error(stream=None) -> tuple[int, int]:
    """Returns (status, raw error word)."""
    v = ctypes.c_uint32(0)
    st = lib().dit_get_device_error(_stream(stream), ctypes.byref(v))
    if st not in (0, DIT_ERR_TIMEOUT):
        raise DitError("dit_get_device_error", st)
    return st, v.value


def dit_clear_device_error(stream=None):
    _call("dit_clear_device_error", _stream(stream))


def dit_set_wait_limit_ns(ns: int):
    _call("dit_set_wait_limit_ns", int(ns))


def dit_selftest_wait_timeout(limit_ns: int, stream=None):
    _call("dit_selftest_wait_timeout", int(limit_ns), _stream(stream))


def dit_rope_table(ids, axes_pairs, theta, rope, stream=None):
    """ids: int32 [S, n_axes] (cuda); rope: float32 [S, sum(axes_pairs), 2] (cuda)."""
    S, n_axes = ids.shape
    arr = (i32 * 3)(*list(axes_pairs) + [0] * (3 - len(axes_pairs)))
    _call("dit_rope_table", _ptr(ids), S, n_axes, arr, float(theta), _ptr(rope), _stream(stream))


def dit_adaln_modulation(vec, W, bias, out, stream=None):
    """vec [B, K] bf16, W [N, K] bf16, bias [N] bf16 or None, out [B, N] fp32."""
    B, K = vec.shape
    N = W.shape[0]
    _call("dit_adaln_modulation", _ptr(vec), vec.stride(0), _ptr(W), W.stride(0), _ptr(bias), _ptr(out),
          out.stride(0), B, N, K, _stream(stream))


def dit_vec_linear(x, W, bias, out, flags=0, stream=None):
    B, K = x.shape
    N = W.shape[0]
    _call("dit_vec_linear", _ptr(x), x.stride(0), _ptr(W), W.stride(0), _ptr(bias), _ptr(out), out.stride(0),
          B, N, K, flags, _stream(stream))


def dit_modulate_norm(x, shift, scale, y, B, S, eps=1e-6, mod_stride=0, stream=None):
    """x, y: bf16 [B*S, D] views (row stride from the tensor); shift/scale fp32 or None."""
    D = x.shape[-1]
    _call("dit_modulate_norm", _ptr(x), x.stride(0), _ptr(shift), _ptr(scale), mod_stride, _ptr(y), y.stride(0),
          B, S, D, float(eps), _stream(stream))


def dit_qk_norm_rope(q, k, q_scale, k_scale, rope, q_out, k_out, B, S, H, eps=1e-6, stream=None):
    """q, k, q_out, k_out: bf16 [B*S, >= H*128] row views with a row stride."""
    _call("dit_qk_norm_rope", _ptr(q), _ptr(k), q.stride(0), _ptr(q_scale), _ptr(k_scale), _ptr(rope),
          _ptr(q_out), _ptr(k_out), q_out.stride(0), B, S, H, 128, float(eps), _stream(stream))


def dit_attention(q, k, v, o, B, Sq, Skv, H, softmax_scale=None, lse=None, stream=None):
    """q, o: bf16 [B*Sq, >= H*128]; k, v: bf16 [B*Skv, >= H*128] (row strides from the tensors)."""
    if softmax_scale is None:
        softmax_scale = 128 ** -0.5
    _call("dit_attention", _ptr(q), _ptr(k), _ptr(v), q.stride(0), k.stride(0), v.stride(0), _ptr(o),
          o.stride(0), _ptr(lse), B, Sq, Skv, H, 128, float(softmax_scale), _stream(stream))


def dit_attention_accumulate(q, k, v, o, lse, B, Sq, Skv, H, softmax_scale=None, stream=None):
    """Merge attention(q, k, v) into the running result (o, lse) in place (one ring hop)."""
    if softmax_scale is None:
        softmax_scale = 128 ** -0.5
    _call("dit_attention_accumulate", _ptr(q), _ptr(k), _ptr(v), q.stride(0), k.stride(0), v.stride(0), _ptr(o),
          o.stride(0), _ptr(lse), B, Sq, Skv, H, 128, float(softmax_scale), _stream(stream))


def dit_set_weight_l2_persist(nbytes):
    """Opt-in L2 residency of the output GEMMs' weights (a process-wide
    persisting L2 set-aside of nbytes on the current device; 0 turns it off)."""
    _call("dit_set_weight_l2_persist", int(nbytes))


def dit_attention_split_workspace(B, Sq, H, n_split):
    """Bytes of device workspace dit_attention_split needs."""
    return lib().dit_attention_split_workspace(B, Sq, H, n_split)


def dit_attention_split(q, k, v, o, B, Sq, Skv, H, n_split, workspace, lse=None, accumulate=False,
                        softmax_scale=None, stream=None):
    """Attention with the keys cut into n_split parts computed side by side
    and merged by log-sum-exp; accumulate merges into the running (o, lse).
    workspace: a uint8 device tensor of dit_attention_split_workspace bytes."""
    if softmax_scale is None:
        softmax_scale = 128 ** -0.5
    _call("dit_attention_split", _ptr(q), _ptr(k), _ptr(v), q.stride(0), k.stride(0), v.stride(0), _ptr(o),
          o.stride(0), _ptr(lse), B, Sq, Skv, H, 128, float(softmax_scale), n_split, int(bool(accumulate)),
          _ptr(workspace), workspace.numel() * workspace.element_size() if workspace is not None else 0,
          _stream(stream))


def dit_selftest_exp2_poly(x, y, stream=None):
    """y = the FMA-pipe 2^x approximation used inside the attention softmax (fp32 device tensors)."""
    _call("dit_selftest_exp2_poly", _ptr(x), _ptr(y), x.numel(), _stream(stream))


def dit_attention_merge(o_parts, lse_parts, o, lse_out, B, Sq, H, stream=None):
    """o = log-sum-exp weighted merge of attention results over disjoint key
    sets; o_parts: bf16 [B*Sq, >= H*128] tensors (one row stride), lse_parts:
    fp32 [B, H, Sq].  o may be one of o_parts, lse_out one of lse_parts."""
    n = len(o_parts)
    if len(lse_parts) != n:
        raise ValueError("o_parts and lse_parts must have the same length")
    ld = o_parts[0].stride(0)
    if any(t.stride(0) != ld for t in o_parts):
        raise ValueError("all parts must share one row stride")
    op = (c_void_p * n)(*[t.data_ptr() for t in o_parts])
    lp = (c_void_p * n)(*[t.data_ptr() for t in lse_parts])
    _call("dit_attention_merge", n, op, lp, ld, _ptr(o), _ptr(lse_out), o.stride(0), B, Sq, H, _stream(stream))


def gemm_args(A, W, C, epi=DIT_EPI_NONE, bias=None, C2=None, split_col=0, gelu_col_begin=0,
              gate=None, gate_stride=0, resid=None, rows_per_batch=0, K=None, qk_cols=0, qk_norm=1,
              qk_eps=1e-6, q_scale=None, k_scale=None, rope=None, rope_rows=0) -> dit_gemm_args:
    """The dit_gemm_args of C[:, :split] (and C2 for the rest) = epilogue(A W^T)."""
    M = A.shape[0]
    N = W.shape[0]
    K = A.shape[1] if K is None else K
    return dit_gemm_args(
        A=_ptr(A), lda=A.stride(0), W=_ptr(W), ldw=W.stride(0), bias=_ptr(bias), C=_ptr(C), ldc=C.stride(0),
        C2=_ptr(C2), ldc2=C2.stride(0) if C2 is not None else 0, split_col=split_col, M=M, N=N, K=K, epi=epi,
        gelu_col_begin=gelu_col_begin, gate=_ptr(gate), gate_stride=gate_stride, resid=_ptr(resid),
        ldr=resid.stride(0) if resid is not None else 0, rows_per_batch=rows_per_batch or M,
        qk_cols=qk_cols, qk_norm=qk_norm, qk_eps=qk_eps, q_scale=_ptr(q_scale), k_scale=_ptr(k_scale),
        rope=_ptr(rope), rope_rows=rope_rows or M)


def dit_gemm_epilogue(A, W, C, epi=DIT_EPI_NONE, bias=None, C2=None, split_col=0, gelu_col_begin=0,
                      gate=None, gate_stride=0, resid=None, rows_per_batch=0, K=None, qk_cols=0, qk_norm=1,
                      qk_eps=1e-6, q_scale=None, k_scale=None, rope=None, rope_rows=0, stream=None):
    """C[:, :split] (and C2 for the rest) = epilogue(A W^T).  A [M, >=K], W [N, >=K]."""
    a = gemm_args(A, W, C, epi, bias, C2, split_col, gelu_col_begin, gate, gate_stride, resid, rows_per_batch, K,
                  qk_cols, qk_norm, qk_eps, q_scale, k_scale, rope, rope_rows)
    _call("dit_gemm_epilogue", ctypes.byref(a), _stream(stream))


def dit_gemm_epilogue_grouped(a: dit_gemm_args, b: dit_gemm_args, stream=None):
    """Two GEMMs (gemm_args) with the same epilogue kind and K in one launch."""
    _call("dit_gemm_epilogue_grouped", ctypes.byref(a), ctypes.byref(b), _stream(stream))


def block_cfg(B, S, D, H, M, n_txt=0, eps=1e-6) -> dit_block_cfg:
    return dit_block_cfg(B=B, S=S, n_txt=n_txt, D=D, H=H, head_dim=128, M=M, eps=eps)


def dit_single_block_workspace(cfg: dit_block_cfg) -> int:
    return lib().dit_single_block_workspace(ctypes.byref(cfg))


def dit_double_block_workspace(cfg: dit_block_cfg) -> int:
    return lib().dit_double_block_workspace(ctypes.byref(cfg))


def dit_video_block_workspace(cfg: dit_block_cfg, n_ctx: int) -> int:
    return lib().dit_video_block_workspace(ctypes.byref(cfg), n_ctx)


def single_weights(w: dict) -> dit_single_weights:
    return dit_single_weights(**{k: _ptr(w[k]) for k, _ in dit_single_weights._fields_})


def double_weights(w: dict) -> dit_double_weights:
    mk = lambda d: dit_stream_weights(**{k: _ptr(d[k]) for k in STREAM_FIELDS})
    return dit_double_weights(txt=mk(w["txt"]), img=mk(w["img"]))


def video_weights(w: dict) -> dit_video_weights:
    return dit_video_weights(**{k: _ptr(w[k]) for k in VIDEO_FIELDS})


def dit_single_block_fwd(cfg, w: dit_single_weights, x, vec, rope, out, ws, stream=None, events=None):
    args = (ctypes.byref(cfg), ctypes.byref(w), _ptr(x), _ptr(vec), _ptr(rope), _ptr(out), _ptr(ws),
            ws.numel() * ws.element_size())
    if events is None:
        _call("dit_single_block_fwd", *args, _stream(stream))
    else:
        arr = (c_void_p * len(events))(*[e.cuda_event for e in events])
        _call("dit_single_block_fwd_profiled", *args, arr, len(events), _stream(stream))


def dit_single_block_fwd_noalloc(cfg, w: dit_single_weights, x, vec, rope, out, stream=None):
    """Single-stream block without a caller workspace: for callers that may
    not allocate device memory.  The intermediates live in a fixed 16 MiB
    array inside the library (shared by all calls; overlapping calls race)."""
    _call("dit_single_block_fwd_noalloc", ctypes.byref(cfg), ctypes.byref(w), _ptr(x), _ptr(vec), _ptr(rope),
          _ptr(out), _stream(stream))


def dit_single_block_host_workspace(cfg: dit_block_cfg) -> int:
    return lib().dit_single_block_host_workspace(ctypes.byref(cfg))


def dit_single_block_fwd_host(cfg, w: dit_single_weights, xs, vecs, outs, rope, ws, stream=None):
    """len(xs) independent single-stream block forwards whose inputs and
    outputs are host tensors (page-locked for overlap); copies in, compute
    and copies out are pipelined inside the library.  The outputs are in
    `outs` once the stream has completed."""
    n = len(xs)
    if len(vecs) != n or len(outs) != n:
        raise ValueError("xs, vecs and outs must have the same length")
    # the copies read and write whole requests: check every host buffer first
    need = {"x": cfg.B * cfg.S * cfg.D * 2, "vec": cfg.B * cfg.D * 2, "out": cfg.B * cfg.S * cfg.D * 2}
    for kind, ts in (("x", xs), ("vec", vecs), ("out", outs)):
        for i, t in enumerate(ts):
            if t.device.type != "cpu" or not t.is_contiguous():
                raise ValueError(f"{kind}[{i}] must be a contiguous host tensor")
            if t.numel() * t.element_size() < need[kind]:
                raise ValueError(f"{kind}[{i}] holds {t.numel() * t.element_size()} bytes, needs {need[kind]}")
    arr = lambda ts: (c_void_p * n)(*[t.data_ptr() for t in ts])
    _call("dit_single_block_fwd_host", ctypes.byref(cfg), ctypes.byref(w), n, arr(xs), arr(vecs), arr(outs),
          _ptr(rope), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream))


def dit_double_block_fwd(cfg, w: dit_double_weights, img, txt, vec, rope, img_out, txt_out, ws, stream=None):
    _call("dit_double_block_fwd", ctypes.byref(cfg), ctypes.byref(w), _ptr(img), _ptr(txt), _ptr(vec),
          _ptr(rope), _ptr(img_out), _ptr(txt_out), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream))


def dit_video_block_fwd(cfg, w: dit_video_weights, x, ctx, n_ctx, vec, rope, out, ws, stream=None):
    _call("dit_video_block_fwd", ctypes.byref(cfg), ctypes.byref(w), _ptr(x), _ptr(ctx), n_ctx, _ptr(vec),
          _ptr(rope), _ptr(out), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream))


class Model:
    """Holds the ctypes structs of a dit_model (weights must stay alive)."""

    def __init__(self, weights: dict, D, H, M, channels=16, txt_dim=4096, t_dim=256, eps=1e-6):
        nd, ns = len(weights["double"]), len(weights["single"])
        self._dbl = (dit_double_weights * max(nd, 1))(*[double_weights(w) for w in weights["double"]])
        self._sgl = (dit_single_weights * max(ns, 1))(*[single_weights(w) for w in weights["single"]])
        kw = {k: _ptr(weights[k]) for k in ("W_img_in", "b_img_in", "W_txt_in", "b_txt_in", "W_t1", "b_t1",
                                             "W_t2", "b_t2", "W_fmod", "b_fmod", "W_out", "b_out")}
        self.c = dit_model(D=D, H=H, head_dim=128, M=M, channels=channels, txt_dim=txt_dim, t_dim=t_dim,
                           n_double=nd, n_single=ns,
                           double_blocks=ctypes.cast(self._dbl, ctypes.POINTER(dit_double_weights)),
                           single_blocks=ctypes.cast(self._sgl, ctypes.POINTER(dit_single_weights)),
                           eps=eps, **kw)


def loop_io(n_txt, grid_h, grid_w, steps, latent_in, txt, ids, latent_out, fresh=None,
            cache_order=1, txt_uncond=None, guidance=1.0, cfg_steps=-1) -> dit_loop_io:
    """fresh: optional sequence of 0/1 per step (1 = run the model).
    txt_uncond: optional unconditional text for classifier-free guidance with
    scale `guidance` on the first cfg_steps steps (< 0: every step)."""
    io = dit_loop_io(n_txt=n_txt, grid_h=grid_h, grid_w=grid_w, steps=steps, latent_in=_ptr(latent_in),
                     txt=_ptr(txt), ids=_ptr(ids), latent_out=_ptr(latent_out), cache_order=cache_order,
                     txt_uncond=_ptr(txt_uncond), guidance=float(guidance), cfg_steps=int(cfg_steps))
    if fresh is not None:
        arr = (ctypes.c_uint8 * steps)(*[1 if f else 0 for f in fresh])
        io._fresh_keep = arr
        io.fresh = ctypes.cast(arr, ctypes.POINTER(ctypes.c_uint8))
    return io


def dit_step_cache_plan(steps: int, fresh, cache_order: int = 1) -> dict:
    """The loop's step-cache plan (host only): per step the kept history slot,
    or for a predicted step the slots and coefficients of v = ca v_a + cb v_b."""
    fr = None if fresh is None else (ctypes.c_uint8 * steps)(*[1 if f else 0 for f in fresh])
    arrs = {k: (i32 * steps)() for k in ("keep_slot", "slot_a", "slot_b")}
    arrs.update({k: (f32 * steps)() for k in ("ca", "cb")})
    _call("dit_step_cache_plan", steps, fr, cache_order, arrs["keep_slot"], arrs["slot_a"], arrs["slot_b"],
          arrs["ca"], arrs["cb"])
    return {k: list(v) for k, v in arrs.items()}


def cached_schedule(steps: int) -> list:
    """Fresh at the first two steps and then every other step: 26 model
    forwards for 50 steps (the count the compile_graph page reports for its
    step cache, §8)."""
    return [1 if (i < 2 or i % 2 == 1) else 0 for i in range(steps)]


def dit_forward_workspace(model: Model, io: dit_loop_io) -> int:
    return lib().dit_forward_workspace(ctypes.byref(model.c), ctypes.byref(io))


def dit_forward_eager(model: Model, io: dit_loop_io, ws, stream=None):
    _call("dit_forward_eager", ctypes.byref(model.c), ctypes.byref(io), _ptr(ws), ws.numel() * ws.element_size(),
          _stream(stream))


class Graph:
    """dit_forward_graph_create / launch / destroy."""

    def __init__(self, model: Model, io: dit_loop_io, ws):
        self._h = c_void_p()
        self._keep = (model, io, ws)
        _call("dit_forward_graph_create", ctypes.byref(model.c), ctypes.byref(io), _ptr(ws),
              ws.numel() * ws.element_size(), ctypes.byref(self._h))

    def launch(self, stream=None):
        _call("dit_forward_graph_launch", self._h, _stream(stream))

    def nodes(self) -> int:
        n = size_t(0)
        _call("dit_forward_graph_nodes", self._h, ctypes.byref(n))
        return n.value

    def destroy(self):
        if self._h:
            _call("dit_forward_graph_destroy", self._h)
            self._h = c_void_p()

    def __del__(self):
        try:
            self.destroy()
        except Exception:
            pass
