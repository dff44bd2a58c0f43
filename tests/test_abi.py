"""CPU checks of the C-ABI library: it loads, exports every symbol the header
declares, and rejects bad arguments before touching the GPU."""
import ctypes

import pytest

import diffusion_transformer_block_flux_b200 as dit
from diffusion_transformer_block_flux_b200 import build


@pytest.fixture(scope="module")
def L():
    build.build()
    return dit.lib()


def test_exports_every_header_symbol(L):
    names = dit.header_functions()
    assert len(names) >= 20
    missing = [n for n in names if not hasattr(L, n)]
    assert not missing, missing
    # and the binding declares a signature for each
    assert set(names) <= set(dit._SIGS), set(names) - set(dit._SIGS)


def test_status_strings_and_version(L):
    assert dit.dit_status_string(0) == "ok"
    assert "aligned" in dit.dit_status_string(3)
    assert dit.dit_status_string(99) == "unknown status"
    assert dit.dit_version() >= 100


def test_argument_validation_is_host_side(L):
    # Null pointers and bad shapes are rejected before any CUDA call.
    assert L.dit_modulate_norm(None, 8, None, None, 0, None, 8, 1, 1, 8, 1e-6, None) == dit.DIT_ERR_INVALID_ARG
    assert L.dit_attention(None, None, None, 128, 128, 128, None, 128, None, 1, 1, 1, 1, 128, 0.1,
                           None) == dit.DIT_ERR_INVALID_ARG
    bad = ctypes.c_void_p(16)
    assert L.dit_attention(bad, bad, bad, 128, 128, 128, bad, 128, None, 1, 1, 1, 1, 64, 0.1,
                           None) == dit.DIT_ERR_UNSUPPORTED
    assert L.dit_qk_norm_rope(bad, bad, 128, None, None, None, bad, bad, 128, 1, 1, 1, 64, 1e-6,
                              None) == dit.DIT_ERR_UNSUPPORTED
    a = dit.dit_gemm_args(A=16, lda=64, W=16, ldw=64, C=16, ldc=64, M=1, N=33, K=64)
    assert L.dit_gemm_epilogue(ctypes.byref(a), None) == dit.DIT_ERR_SHAPE
    a = dit.dit_gemm_args(A=24, lda=64, W=16, ldw=64, C=16, ldc=64, M=1, N=64, K=64)
    assert L.dit_gemm_epilogue(ctypes.byref(a), None) == dit.DIT_ERR_ALIGNMENT
    assert L.dit_gemm_epilogue(None, None) == dit.DIT_ERR_INVALID_ARG
    assert L.dit_set_wait_limit_ns(0) == dit.DIT_ERR_INVALID_ARG
    assert L.dit_selftest_wait_timeout(0, None) == dit.DIT_ERR_INVALID_ARG


def test_workspace_sizes(L):
    cfg = dit.block_cfg(1, 4608, 3072, 24, 12288, n_txt=512)
    ws = dit.dit_single_block_workspace(cfg)
    # mod + y + qkv + [attn | mlp]
    expect = 3 * 3072 * 4 + 4608 * 3072 * 2 * (1 + 3) + 4608 * (3072 + 12288) * 2
    assert expect <= ws <= expect + 4 * 256
    assert dit.dit_double_block_workspace(cfg) > 0
    assert dit.dit_video_block_workspace(dit.block_cfg(1, 28350, 1536, 12, 8960), 512) > 0
    bad = dit.block_cfg(1, 4608, 3072, 24, 12288)
    bad.head_dim = 64
    assert dit.dit_single_block_workspace(bad) == 0


def test_block_call_rejects_small_workspace(L):
    cfg = dit.block_cfg(1, 256, 384, 3, 1536)
    w = dit.dit_single_weights(*([16] * 8))
    st = L.dit_single_block_fwd(ctypes.byref(cfg), ctypes.byref(w), 16, 16, 16, 16, 256, 10, None)
    assert st == dit.DIT_ERR_WORKSPACE


def test_host_pipeline_validation(L):
    cfg = dit.block_cfg(1, 256, 384, 3, 1536)
    w = dit.dit_single_weights(*([16] * 8))
    one = (ctypes.c_void_p * 1)(16)
    nul = (ctypes.c_void_p * 1)(None)
    need = dit.dit_single_block_host_workspace(cfg)
    # block workspace + two staging slots of x, vec and out
    assert need >= dit.dit_single_block_workspace(cfg) + 2 * (2 * 256 * 384 * 2 + 384 * 2)
    f = L.dit_single_block_fwd_host
    assert f(ctypes.byref(cfg), ctypes.byref(w), 0, one, one, one, 16, 256, need, None) == dit.DIT_ERR_INVALID_ARG
    assert f(ctypes.byref(cfg), ctypes.byref(w), 1, one, nul, one, 16, 256, need, None) == dit.DIT_ERR_INVALID_ARG
    assert f(ctypes.byref(cfg), ctypes.byref(w), 1, one, one, one, 16, 256, need - 1, None) == dit.DIT_ERR_WORKSPACE
    assert f(ctypes.byref(cfg), ctypes.byref(w), 1, one, one, one, 16, 264, need, None) == dit.DIT_ERR_ALIGNMENT


def test_binding_struct_layouts_match_the_library(L):
    """Every ctypes struct of the binding has the size the library was
    compiled with (a field added to the header but not to the binding, or
    the other way round, fails here)."""
    structs = [dit.dit_gemm_args, dit.dit_block_cfg, dit.dit_single_weights, dit.dit_stream_weights,
               dit.dit_double_weights, dit.dit_video_weights, dit.dit_model, dit.dit_loop_io]
    for i, st in enumerate(structs):
        assert L.dit_abi_struct_size(i) == ctypes.sizeof(st), (st.__name__, L.dit_abi_struct_size(i),
                                                               ctypes.sizeof(st))
    assert L.dit_abi_struct_size(len(structs)) == 0


@pytest.mark.parametrize("order", [0, 1])
@pytest.mark.parametrize("fresh", [[1, 1, 0, 1, 0, 0], [1, 0, 0, 1, 0], [1] * 5, "cached50"])
def test_step_cache_plan_follows_the_definition(L, order, fresh):
    """The loop's host bookkeeping of the step cache: a predicted step reads the
    kept velocities of the two newest fresh steps a (newest) and b, with
    v = v_a + (t - t_a)(v_a - v_b)/(t_a - t_b) for order 1 (v_a alone for
    order 0 or while only one exists); a fresh step keeps its velocity in the
    slot not holding the newest one."""
    if fresh == "cached50":
        fresh = dit.cached_schedule(50)
    n = len(fresh)
    p = dit.dit_step_cache_plan(n, fresh, order)
    t = [1.0 - i / n for i in range(n)]
    done = []  # fresh steps so far
    for i in range(n):
        if fresh[i]:
            assert p["keep_slot"][i] in (0, 1) and p["slot_a"][i] == -1 and p["slot_b"][i] == -1
            if done:
                assert p["keep_slot"][i] != p["keep_slot"][done[-1]]  # the newest stays readable
            done.append(i)
            continue
        a = done[-1]
        assert p["keep_slot"][i] == -1 and p["slot_a"][i] == p["keep_slot"][a]
        if order == 1 and len(done) >= 2:
            b = done[-2]
            r = (t[i] - t[a]) / (t[a] - t[b])
            assert p["slot_b"][i] == p["keep_slot"][b]
            assert abs(p["ca"][i] - (1 + r)) <= 1e-6 * abs(1 + r) and abs(p["cb"][i] + r) <= 1e-6 * abs(r)
        else:
            assert p["slot_b"][i] == -1 and p["ca"][i] == 1.0 and p["cb"][i] == 0.0


def test_step_cache_plan_without_cache_and_validation(L):
    p = dit.dit_step_cache_plan(4, None, 1)
    assert p["keep_slot"] == [-1] * 4 and p["slot_a"] == [-1] * 4
    bad = (ctypes.c_uint8 * 3)(0, 1, 1)
    i3 = (ctypes.c_int * 3)()
    f3 = (ctypes.c_float * 3)()
    assert L.dit_step_cache_plan(3, bad, 1, i3, i3, i3, f3, f3) == dit.DIT_ERR_INVALID_ARG
    assert L.dit_step_cache_plan(3, None, 2, i3, i3, i3, f3, f3) == dit.DIT_ERR_INVALID_ARG


def _fake_model(nd, ns, D=256, H=2, M=512):
    """A dit_model of placeholder (never dereferenced) pointers: enough for the
    host-side validation and workspace query."""
    P = 256
    dbl = (dit.dit_double_weights * max(nd, 1))(*[dit.dit_double_weights(
        txt=dit.dit_stream_weights(*([P] * 12)), img=dit.dit_stream_weights(*([P] * 12))) for _ in range(nd)])
    sgl = (dit.dit_single_weights * max(ns, 1))(*[dit.dit_single_weights(*([P] * 8)) for _ in range(ns)])
    m = dit.dit_model(D=D, H=H, head_dim=128, M=M, channels=16, txt_dim=64, t_dim=256, n_double=nd, n_single=ns,
                      double_blocks=ctypes.cast(dbl, ctypes.POINTER(dit.dit_double_weights)),
                      single_blocks=ctypes.cast(sgl, ctypes.POINTER(dit.dit_single_weights)), eps=1e-6,
                      **{k: P for k in ("W_img_in", "b_img_in", "W_txt_in", "b_txt_in", "W_t1", "b_t1", "W_t2",
                                        "b_t2", "W_fmod", "b_fmod", "W_out", "b_out")})
    m._keep = (dbl, sgl)
    return m


def _fake_io(steps=6, **kw):
    io = dit.dit_loop_io(n_txt=16, grid_h=4, grid_w=6, steps=steps, latent_in=256, txt=256, ids=256, latent_out=256,
                         cache_order=1, guidance=1.0, cfg_steps=-1)
    for k, v in kw.items():
        setattr(io, k, v)
    return io


def test_loop_workspace_query_validates_on_the_host(L):
    m = _fake_model(2, 2)
    ws = L.dit_forward_workspace(ctypes.byref(m), ctypes.byref(_fake_io()))
    assert ws > 0
    # the per-step modulation buffer (every block's vectors, fp32) is part of it
    m0 = _fake_model(0, 0)
    ws0 = L.dit_forward_workspace(ctypes.byref(m0), ctypes.byref(_fake_io()))
    assert ws - ws0 >= 4 * 256 * (12 * 2 + 3 * 2)
    # guidance: an unconditional text with a finite scale is fine, a NaN scale is not
    assert L.dit_forward_workspace(ctypes.byref(m), ctypes.byref(_fake_io(txt_uncond=256, guidance=3.0))) == ws
    assert L.dit_forward_workspace(ctypes.byref(m), ctypes.byref(_fake_io(txt_uncond=256,
                                                                          guidance=float("nan")))) == 0
    # step cache: the first step must run the model; orders 0 and 1 only
    bad = (ctypes.c_uint8 * 6)(0, 1, 1, 1, 1, 1)
    assert L.dit_forward_workspace(ctypes.byref(m), ctypes.byref(_fake_io(
        fresh=ctypes.cast(bad, ctypes.POINTER(ctypes.c_uint8))))) == 0
    assert L.dit_forward_workspace(ctypes.byref(m), ctypes.byref(_fake_io(cache_order=2))) == 0
    assert L.dit_forward_workspace(ctypes.byref(m), ctypes.byref(_fake_io(steps=0))) == 0
    assert L.dit_forward_workspace(ctypes.byref(m), ctypes.byref(_fake_io(txt=None))) == 0


def test_new_entry_points_reject_bad_arguments_on_the_host(L):
    p = ctypes.c_void_p(256)
    one = (ctypes.c_void_p * 1)(256)
    nine = (ctypes.c_void_p * 9)(*([256] * 9))
    # merge: 1..8 parts, heads and batch in range, 16-byte aligned rows
    assert L.dit_attention_merge(0, one, one, 128, p, None, 128, 1, 4, 1, None) == dit.DIT_ERR_INVALID_ARG
    assert L.dit_attention_merge(9, nine, nine, 128, p, None, 128, 1, 4, 1, None) == dit.DIT_ERR_INVALID_ARG
    assert L.dit_attention_merge(1, one, one, 64, p, None, 128, 1, 4, 1, None) == dit.DIT_ERR_SHAPE
    assert L.dit_attention_merge(1, one, one, 130, p, None, 130, 1, 4, 1, None) == dit.DIT_ERR_ALIGNMENT
    assert L.dit_attention_merge(1, one, one, 128, ctypes.c_void_p(258), None, 128, 1, 4, 1,
                                 None) == dit.DIT_ERR_ALIGNMENT
    assert L.dit_attention_merge(1, one, one, 128, p, None, 128, 70000, 4, 1, None) == dit.DIT_ERR_SHAPE
    # exp2 self test
    assert L.dit_selftest_exp2_poly(None, p, 4, None) == dit.DIT_ERR_INVALID_ARG
    assert L.dit_selftest_exp2_poly(p, p, 0, None) == dit.DIT_ERR_INVALID_ARG


def test_host_pipeline_binding_checks_host_buffers(L):
    import torch
    cfg = dit.block_cfg(1, 8, 128, 1, 256)
    w = dit.dit_single_weights(*([256] * 8))
    ok = torch.empty((8, 128), dtype=torch.bfloat16)
    v = torch.empty((1, 128), dtype=torch.bfloat16)
    ws = torch.empty(16, dtype=torch.uint8)
    with pytest.raises(ValueError, match="same length"):
        dit.dit_single_block_fwd_host(cfg, w, [ok], [v, v], [ok], None, ws)
    with pytest.raises(ValueError, match="needs"):
        dit.dit_single_block_fwd_host(cfg, w, [ok[:4]], [v], [ok], None, ws)
    with pytest.raises(ValueError, match="contiguous"):
        dit.dit_single_block_fwd_host(cfg, w, [ok], [v], [torch.empty((128, 8), dtype=torch.bfloat16).t()], None, ws)


def test_noalloc_reports_the_same_status_as_the_workspace_call(L):
    """For a configuration the block rejects, the allocation-free call returns
    the status the workspace call returns (both checks run on the host before
    anything is enqueued); a valid but too large configuration is a workspace
    error."""
    w = dit.dit_single_block_workspace
    weights = dit.dit_single_weights()
    for cfg in (dit.block_cfg(1, 256, 384, 2, 1536),            # D != H * 128
                dit.block_cfg(1, 256, 384, 3, 1536, eps=float("nan")),
                dit.block_cfg(0, 256, 384, 3, 1536),
                dit.block_cfg(1, 256, 384, 3, 100)):              # M not a multiple of 32
        assert w(cfg) == 0
        ref = L.dit_single_block_fwd(ctypes.byref(cfg), ctypes.byref(weights), None, None, None, None, None, 0, None)
        got = L.dit_single_block_fwd_noalloc(ctypes.byref(cfg), ctypes.byref(weights), None, None, None, None, None)
        assert ref != dit.DIT_OK and got == ref
    assert L.dit_single_block_fwd_noalloc(None, ctypes.byref(weights), None, None, None, None, None) == \
        dit.DIT_ERR_INVALID_ARG
    big = dit.block_cfg(1, 4608, 3072, 24, 12288)
    assert L.dit_single_block_fwd_noalloc(ctypes.byref(big), ctypes.byref(weights), None, None, None, None,
                                          None) == dit.DIT_ERR_WORKSPACE


def test_split_attention_and_grouped_gemm_validate_on_the_host(L):
    """The key-split attention's workspace query is plain arithmetic (one bf16
    partial result and one fp32 lse per split, each 256-byte aligned, at most
    four splits); bad split counts, a missing or misaligned workspace and
    mismatched grouped GEMM jobs are rejected before any CUDA call."""
    def a256(n):
        return (n + 255) // 256 * 256
    B, Sq, H = 2, 577, 3
    for n in (1, 2, 3, 4, 7):
        k = min(n, 4)
        assert L.dit_attention_split_workspace(B, Sq, H, n) == k * a256(B * Sq * H * 128 * 2) + k * a256(B * H * Sq * 4)
    for bad in ((0, Sq, H, 2), (B, 0, H, 2), (B, Sq, 0, 2), (B, Sq, H, 0)):
        assert L.dit_attention_split_workspace(*bad) == 0
    p = ctypes.c_void_p(256)
    ws = L.dit_attention_split_workspace(1, 64, 1, 2)

    def split(n_split, accumulate=0, lse=p, workspace=p, nbytes=ws, Skv=1000, B=1):
        return L.dit_attention_split(p, p, p, 128, 128, 128, p, 128, lse, B, 64, Skv, 1, 128, 0.1, n_split,
                                     accumulate, workspace, nbytes, None)
    assert split(0) == dit.DIT_ERR_INVALID_ARG
    assert split(5) == dit.DIT_ERR_INVALID_ARG
    assert split(2, accumulate=1, lse=None) == dit.DIT_ERR_INVALID_ARG
    assert split(2, B=0) == dit.DIT_ERR_SHAPE
    # 1000 keys are 8 key tiles: two splits need the workspace
    assert split(2, workspace=None) == dit.DIT_ERR_WORKSPACE
    assert split(2, nbytes=ws - 1) == dit.DIT_ERR_WORKSPACE
    assert split(2, workspace=ctypes.c_void_p(272)) == dit.DIT_ERR_ALIGNMENT
    # grouped GEMM: both jobs valid, same epilogue and the same K
    g1 = dit.dit_gemm_args(A=256, lda=64, W=256, ldw=64, C=256, ldc=64, M=256, N=64, K=64)
    g2 = dit.dit_gemm_args(A=256, lda=128, W=256, ldw=128, C=256, ldc=64, M=256, N=64, K=128)
    assert L.dit_gemm_epilogue_grouped(None, ctypes.byref(g1), None) == dit.DIT_ERR_INVALID_ARG
    assert L.dit_gemm_epilogue_grouped(ctypes.byref(g1), ctypes.byref(g2), None) == dit.DIT_ERR_INVALID_ARG
    bad = dit.dit_gemm_args(A=256, lda=64, W=256, ldw=64, C=256, ldc=64, M=1, N=33, K=64)
    assert L.dit_gemm_epilogue_grouped(ctypes.byref(g1), ctypes.byref(bad), None) == dit.DIT_ERR_SHAPE
