"""The workspace-free block entry point, klein_block_forward_static.

Some callers cannot call cudaMalloc: a plug-in running inside a host
application that owns all device memory through its own pool and forbids
allocating around it, or code on a latency-critical path where a device
allocation (which may synchronise the device) is not allowed. This entry
point keeps its scratch in a fixed array inside the library instead. It runs
the same kernels on the same data as klein_block_forward with a caller
workspace, so its results must equal that path's bit for bit, call after
call, although consecutive calls reuse (and inherit the contents of) the one
array.

Named so that pytest collects it last."""
import ctypes

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import klein_inputs as ki  # noqa: E402
from gpu_util import host, max_err_ratio, to_f32, upload_block, workspace  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kb():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from conftest import ensure_built
    ensure_built()
    import latent_flow_matching_joint_b200 as kb
    return kb


def test_static_scratch_block_matches_workspace_block(kb):
    w = upload_block(ki.block_weights(0, "joint.0"))
    n_txt, gh, gw = 80, 8, 8              # 80 text + 8x8 image tokens, batch 1
    n = n_txt + gh * gw
    x = ki.tokens(1, "no_alloc", 1, n)
    mod = to_f32(ki.modulation_vectors(1, "no_alloc"))
    pos = torch.empty((n, 4), dtype=torch.float32, device="cuda")
    kb.klein_positions(kb.make_seq(1, n_txt, gh, gw), pos)

    ref = to_f32(x)
    ws = workspace(kb.klein_block_workspace_size(1, n))
    kb.klein_block_forward(w, ref, n_txt, gh * gw, pos, mod, ws)
    torch.cuda.synchronize()
    expect = host(ref)

    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    bw = kb.block_weights(w)
    for call in range(2):                 # the second call reuses the first call's scratch
        got = to_f32(x)
        rc = kb.lib.klein_block_forward_static(ctypes.byref(bw), ctypes.c_void_p(got.data_ptr()), 1, n, 0, n, n_txt,
                                               gh * gw, ctypes.c_void_p(pos.data_ptr()),
                                               ctypes.c_void_p(mod.data_ptr()), stream)
        assert rc == 0, kb.lib.klein_last_error()
        torch.cuda.synchronize()
        g = host(got)
        assert np.all(np.isfinite(g)), call
        np.testing.assert_array_equal(g, expect)
    assert kb.klein_device_status()[0] == 0


def test_static_scratch_row_range_with_mixed_modes(kb):
    # a stage-1 style call on a row range that starts inside the sequence:
    # rows 80..143 of 80 text + 5x8 image + 4x6 reference tokens (image rows
    # take mode 1, reference rows mode 2, by global row index), batch 2 x 64
    # rows (128 after rounding up); bit-identical to the workspace path
    w = upload_block(ki.block_weights(0, "joint.1"))
    n_txt, n_img, n_ref = 80, 40, 24
    n = n_txt + n_img + n_ref
    x = ki.tokens(1, "no_alloc.range", 2, n)
    mod = to_f32(ki.modulation_vectors(1, "no_alloc.range"))
    pos = torch.empty((n, 4), dtype=torch.float32, device="cuda")
    kb.klein_positions(kb.make_seq(2, n_txt, 5, 8, refs=((4, 6),)), pos)
    ref = to_f32(x)
    ws = workspace(kb.klein_block_workspace_size(2, n - n_txt))
    kb.klein_block_forward(w, ref, n_txt, n_img, pos, mod, ws, row0=n_txt, rows=n - n_txt)
    torch.cuda.synchronize()
    expect = host(ref)
    assert max_err_ratio(expect[:, :n_txt], x[:, :n_txt].astype(np.float64)) == 0.0   # rows outside the range kept
    for _ in range(2):
        got = to_f32(x)
        kb.klein_block_forward_static(w, got, n_txt, n_img, pos, mod, row0=n_txt, rows=n - n_txt)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(host(got), expect)
    assert kb.klein_device_status()[0] == 0


def test_static_scratch_rejects_oversized_calls(kb):
    w = upload_block(ki.block_weights(0, "joint.0"))
    n = 300                               # 300 rows round up to 384 > 256
    x = torch.zeros((1, n, ki.DIM), dtype=torch.float32, device="cuda")
    pos = torch.zeros((n, 4), dtype=torch.float32, device="cuda")
    mod = torch.zeros((3, 3, ki.DIM), dtype=torch.float32, device="cuda")
    with pytest.raises(kb.KleinError) as e:
        kb.klein_block_forward_static(w, x, 100, 200, pos, mod)
    assert e.value.name == "KLEIN_ERR_WORKSPACE"
    with pytest.raises(kb.KleinError) as e:   # batch 2 x 200 rows also exceeds it
        kb.klein_block_forward_static(w, torch.zeros((2, 200, ki.DIM), device="cuda"), 100, 100, pos, mod)
    assert e.value.name == "KLEIN_ERR_WORKSPACE"


def test_static_scratch_fp8_block_at_the_size_limit(kb):
    # rowwise FP8 weights, batch 2 x 128 rows = the array's limit of 256
    # rows; the per-row activation scales live in the same fixed array, so
    # the result is the workspace path's, bit for bit (same kernels, same
    # reduction orders)
    w = kb.quantize_block_e4m3(upload_block(ki.block_weights(0, "joint.0")))
    n_txt, gh, gw = 64, 8, 8
    n = n_txt + gh * gw                   # 128 rows
    x = ki.tokens(1, "no_alloc.fp8", 2, n)
    mod = to_f32(ki.modulation_vectors(1, "no_alloc.fp8"))
    pos = torch.empty((n, 4), dtype=torch.float32, device="cuda")
    kb.klein_positions(kb.make_seq(2, n_txt, gh, gw), pos)
    ref = to_f32(x)
    ws = workspace(kb.klein_block_workspace_size(2, n))
    kb.klein_block_forward(w, ref, n_txt, gh * gw, pos, mod, ws)
    for _ in range(2):
        got = to_f32(x)
        kb.klein_block_forward_static(w, got, n_txt, gh * gw, pos, mod)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(host(got), host(ref))
    assert kb.klein_device_status()[0] == 0


def test_static_scratch_nvfp4_block_at_the_size_limit(kb):
    # NVFP4 weights, batch 2 x 128 rows = the array's limit of 256 rows; the
    # block scales of both GEMM inputs are laid out per batch item over 256
    # rows (the GEMM's row tile), which the fixed array reserves as well, so
    # the result is the workspace path's, bit for bit
    w = kb.quantize_block_nvfp4(upload_block(ki.block_weights(0, "joint.0")))
    n_txt, gh, gw = 64, 8, 8
    n = n_txt + gh * gw                   # 128 rows
    x = ki.tokens(1, "no_alloc.nvfp4", 2, n)
    mod = to_f32(ki.modulation_vectors(1, "no_alloc.nvfp4"))
    pos = torch.empty((n, 4), dtype=torch.float32, device="cuda")
    kb.klein_positions(kb.make_seq(2, n_txt, gh, gw), pos)
    ref = to_f32(x)
    ws = workspace(kb.klein_block_workspace_size(2, n))
    kb.klein_block_forward(w, ref, n_txt, gh * gw, pos, mod, ws)
    for _ in range(2):
        got = to_f32(x)
        kb.klein_block_forward_static(w, got, n_txt, gh * gw, pos, mod)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(host(got), host(ref))
    assert kb.klein_device_status()[0] == 0
