"""CPU tests of the C-ABI library: it loads, exports every symbol the header
declares, and its host-only functions (schedule, padding, sequence counts,
argument checks) agree with the oracle. No device work is issued."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle as o

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def kb():
    from conftest import ensure_built
    ensure_built()
    import latent_flow_matching_joint_b200 as kb
    return kb


def header_functions():
    text = open(os.path.join(ROOT, "include", "klein.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(klein_[a-z0-9_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol(kb):
    declared = header_functions()
    assert len(declared) >= 20
    for name in declared:
        assert hasattr(kb.lib, name), name
    # the binding wraps exactly the declared C functions
    assert sorted(kb.EXPORTED) == declared


def test_schedule_matches_oracle(kb):
    for steps in (1, 4, 16, 50):
        got = np.array(kb.klein_sigma_schedule(steps))
        np.testing.assert_allclose(got, o.sigma_schedule(steps), rtol=0, atol=6e-8)
    assert kb.klein_sigma_schedule(16)[-1] == 0.0


def test_pad_text_len_matches_oracle(kb):
    for n in (0, 1, 79, 80, 81, 160, 512, 1000):
        assert kb.klein_pad_text_len(n) == o.pad_text_len(n)
    assert kb.klein_pad_text_len(-1) == -1


def test_seq_tokens(kb):
    s = kb.make_seq(1, 512, 64, 64)
    assert kb.klein_seq_tokens(s) == (4096, 0, 4608)
    s = kb.make_seq(1, 512, 64, 64, refs=[(64, 64)])
    assert kb.klein_seq_tokens(s) == (4096, 4096, 8704)
    s = kb.make_seq(2, 560, 128, 128)
    assert kb.klein_seq_tokens(s) == (16384, 0, 16944)
    assert kb.klein_seq_tokens(kb.make_seq(1, 80, 8, 8)) == (64, 0, 144)


def test_seq_errors(kb):
    for bad in (kb.make_seq(0, 10, 2, 2), kb.make_seq(1, 0, 2, 2), kb.make_seq(1, 5, 0, 2)):
        with pytest.raises(kb.KleinError) as e:
            kb.klein_seq_tokens(bad)
        assert e.value.name == "KLEIN_ERR_SHAPE"
    s = kb.make_seq(1, 5, 2, 2)
    s.n_refs = 11
    with pytest.raises(kb.KleinError):
        kb.klein_seq_tokens(s)


def test_workspace_sizes_grow(kb):
    a = kb.klein_block_workspace_size(1, 144)
    b = kb.klein_block_workspace_size(1, 4608)
    c = kb.klein_block_workspace_size(2, 4608)
    assert 0 < a < b < c
    assert kb.klein_block_workspace_size(0, 10) == 0
    s1 = kb.klein_stack_workspace_size(kb.make_seq(1, 512, 64, 64))
    assert s1 > kb.klein_block_workspace_size(1, 4608)


def test_argument_errors_before_any_launch(kb):
    bw = kb.KleinBlockWeights(None, None, None, None)
    rc = kb.lib.klein_block_forward(ctypes.byref(bw), None, 1, 10, 0, 10, 5, 5, None, None, None, 0, None)
    assert kb.STATUS[rc] == "KLEIN_ERR_INVALID_ARG"
    assert b"incomplete" in kb.lib.klein_last_error()
    # misaligned weights
    bw = kb.KleinBlockWeights(16, 18, 32, 48)
    rc = kb.lib.klein_block_forward(ctypes.byref(bw), None, 1, 10, 0, 10, 5, 5, None, None, None, 0, None)
    assert kb.STATUS[rc] == "KLEIN_ERR_ALIGN"
    # bad range
    bw = kb.KleinBlockWeights(16, 32, 48, 64)
    rc = kb.lib.klein_block_forward(ctypes.byref(bw), 256, 1, 10, 5, 10, 5, 5, 256, 256, 256, 1 << 30, None)
    assert kb.STATUS[rc] == "KLEIN_ERR_SHAPE"
    # workspace too small
    rc = kb.lib.klein_block_forward(ctypes.byref(bw), 256, 1, 10, 0, 10, 5, 5, 256, 256, 256, 1024, None)
    assert kb.STATUS[rc] == "KLEIN_ERR_WORKSPACE"
    # stream sizes that do not fit the sequence (6 text + 5 image rows > 10)
    for fn, extra in ((kb.lib.klein_block_forward, (256, 1 << 30)), (kb.lib.klein_block_forward_static, ())):
        rc = fn(ctypes.byref(bw), 256, 1, 10, 0, 10, 6, 5, 256, 256, *extra, None)
        assert kb.STATUS[rc] == "KLEIN_ERR_SHAPE"
        assert b"exceeds n_total" in kb.lib.klein_last_error()
        rc = fn(ctypes.byref(bw), 256, 1, 10, 0, 10, -1, 5, 256, 256, *extra, None)
        assert kb.STATUS[rc] == "KLEIN_ERR_SHAPE"
    rc = kb.lib.klein_op_gemm(256, 256, 256, 10, 100, 64, None)
    assert kb.STATUS[rc] == "KLEIN_ERR_SHAPE"
    rc = kb.lib.klein_op_euler(256, 256, None, 6, ctypes.c_float(0.1), ctypes.c_float(1.0), None,
                               ctypes.c_float(0.0), None)
    assert kb.STATUS[rc] == "KLEIN_ERR_SHAPE"
    assert kb.lib.klein_wait_probe(0, None) == -1


def test_model_create_validation(kb):
    d = kb.KleinModelDesc()
    d.n_stage1, d.n_joint = 0, 0
    h = ctypes.c_void_p()
    rc = kb.lib.klein_model_create(ctypes.byref(h), ctypes.byref(d))
    assert kb.STATUS[rc] == "KLEIN_ERR_INVALID_ARG"


def test_fp8_argument_errors_before_any_launch(kb):
    q = kb.lib.klein_quantize_rowwise_e4m3
    rc = q(None, 4, 16, 256, 512, None)
    assert kb.STATUS[rc] == "KLEIN_ERR_INVALID_ARG"
    rc = q(256, 4, 12, 4096, 8192, None)                 # cols not a multiple of 8
    assert kb.STATUS[rc] == "KLEIN_ERR_SHAPE"
    rc = q(256, 4, 12296, 1 << 20, 1 << 21, None)        # cols beyond 12288
    assert kb.STATUS[rc] == "KLEIN_ERR_SHAPE"
    rc = q(264, 4, 16, 4096, 8192, None)                 # src not 16-byte aligned
    assert kb.STATUS[rc] == "KLEIN_ERR_ALIGN"
    rc = q(4096, 4, 16, 4096 + 64, 8192, None)           # codes overlap src
    assert kb.STATUS[rc] == "KLEIN_ERR_INVALID_ARG"
    g = kb.lib.klein_op_gemm_e4m3
    rc = g(256, 512, 1024, 2048, 4096, 10, 200, 128, None)  # N not a multiple of 256
    assert kb.STATUS[rc] == "KLEIN_ERR_SHAPE"
    rc = g(256, 512, 1024, 2048, 4096, 10, 256, 96, None)   # K not a multiple of 128
    assert kb.STATUS[rc] == "KLEIN_ERR_SHAPE"
    # FP8 block weights need both scales
    bw = kb.KleinBlockWeights(16, 32, 48, 64, 80, None)
    rc = kb.lib.klein_block_forward(ctypes.byref(bw), 256, 1, 10, 0, 10, 5, 5, 256, 256, 256, 1 << 30, None)
    assert kb.STATUS[rc] == "KLEIN_ERR_INVALID_ARG"
    assert b"w_in_scale and w_out_scale" in kb.lib.klein_last_error()


def _fake_model(kb, distilled=True):
    """A model handle over aligned placeholder addresses: it passes
    klein_model_create (which checks presence and alignment only) and serves
    the argument checks below, each of which must fail before any launch
    could read a weight."""
    d = kb.KleinModelDesc()
    d.n_stage1, d.n_joint = 0, 1
    bw = kb.KleinBlockWeights(1 << 12, 2 << 12, 3 << 12, 4 << 12)
    d.joint = ctypes.cast(ctypes.pointer(bw), ctypes.c_void_p)
    d.img_in, d.t_mlp1, d.t_mlp2, d.final_mod, d.final_out = 5 << 12, 6 << 12, 7 << 12, 8 << 12, 9 << 12
    if distilled:
        d.tt_mlp1, d.tt_mlp2 = 10 << 12, 11 << 12
    for st in range(2):
        for m in range(2):
            d.mod[st][m] = (12 + 2 * st + m) << 12
    h = ctypes.c_void_p()
    assert kb.lib.klein_model_create(ctypes.byref(h), ctypes.byref(d)) == 0
    return h, bw          # the caller keeps bw alive: the model borrows it


def test_denoise_and_stack_argument_errors(kb):
    h, _bw = _fake_model(kb)
    seq = kb.make_seq(1, 80, 8, 8)
    seq2 = kb.make_seq(2, 80, 8, 8)
    lat, txt, ws, big = 1 << 20, 2 << 20, 3 << 20, 1 << 40
    den = kb.lib.klein_denoise

    def st(rc):
        return kb.STATUS[rc]

    try:
        assert st(den(None, lat, txt, None, 4, 1.0, 6.93, ctypes.byref(seq), None, 0, ws, big, None)) == \
            "KLEIN_ERR_INVALID_ARG"
        assert b"model is NULL" in kb.lib.klein_last_error()
        assert st(den(h, lat, txt, None, 4, 1.0, 6.93, None, None, 0, ws, big, None)) == "KLEIN_ERR_INVALID_ARG"
        bad = kb.make_seq(1, 80, 8, 8)
        bad.batch = 0
        assert st(den(h, lat, txt, None, 4, 1.0, 6.93, ctypes.byref(bad), None, 0, ws, big, None)) == \
            "KLEIN_ERR_SHAPE"
        assert st(den(h, None, txt, None, 4, 1.0, 6.93, ctypes.byref(seq), None, 0, ws, big, None)) == \
            "KLEIN_ERR_INVALID_ARG"
        assert st(den(h, lat + 4, txt, None, 4, 1.0, 6.93, ctypes.byref(seq), None, 0, ws, big, None)) == \
            "KLEIN_ERR_ALIGN"
        # a reference in the sequence, but no reference weights in the model
        rseq = kb.make_seq(1, 80, 8, 8, ((4, 4),))
        assert st(den(h, lat, txt, 4 << 20, 4, 1.0, 6.93, ctypes.byref(rseq), None, 0, ws, big, None)) == \
            "KLEIN_ERR_INVALID_ARG"
        assert b"reference weights" in kb.lib.klein_last_error()
        need = kb.lib.klein_stack_workspace_size(ctypes.byref(seq))
        assert st(den(h, lat, txt, None, 4, 1.0, 6.93, ctypes.byref(seq), None, 0, ws, need - 1, None)) == \
            "KLEIN_ERR_WORKSPACE"
        for steps in (0, 1001):
            assert st(den(h, lat, txt, None, steps, 1.0, 6.93, ctypes.byref(seq), None, 0, ws, big, None)) == \
                "KLEIN_ERR_INVALID_ARG"
        # guidance needs the (cond, uncond) pair as batch 2, and only then
        assert st(den(h, lat, txt, None, 4, 3.5, 6.93, ctypes.byref(seq), None, 0, ws, big, None)) == \
            "KLEIN_ERR_SHAPE"
        assert st(den(h, lat, txt, None, 4, 1.0, 6.93, ctypes.byref(seq2), None, 0, ws, big, None)) == \
            "KLEIN_ERR_SHAPE"
        assert st(den(h, lat, txt, None, 4, 1.0, 6.93, ctypes.byref(seq), lat + 8, 0, ws, big, None)) == \
            "KLEIN_ERR_ALIGN"
        assert st(den(h, lat, txt, None, 4, 1.0, 0.0, ctypes.byref(seq), None, 0, ws, big, None)) == \
            "KLEIN_ERR_INVALID_ARG"
        assert b"shift" in kb.lib.klein_last_error()
        sf = kb.lib.klein_stack_forward
        assert st(sf(h, lat, txt, None, ctypes.c_float(0.5), ctypes.c_float(0.4), ctypes.byref(seq), None, ws,
                     big, None)) == "KLEIN_ERR_ALIGN"
        assert st(sf(h, lat, txt, None, ctypes.c_float(0.5), ctypes.c_float(0.4), ctypes.byref(seq), 5 << 20, ws,
                     need - 16, None)) == "KLEIN_ERR_WORKSPACE"
    finally:
        kb.lib.klein_model_destroy(h)


def test_schedule_and_positions_argument_errors(kb):
    out = (ctypes.c_float * 8)()
    assert kb.STATUS[kb.lib.klein_sigma_schedule(0, 6.93, out)] == "KLEIN_ERR_INVALID_ARG"
    assert kb.STATUS[kb.lib.klein_sigma_schedule(4, -1.0, out)] == "KLEIN_ERR_INVALID_ARG"
    assert kb.STATUS[kb.lib.klein_sigma_schedule(4, 6.93, None)] == "KLEIN_ERR_INVALID_ARG"
    seq = kb.make_seq(1, 80, 8, 8)
    assert kb.STATUS[kb.lib.klein_positions(ctypes.byref(seq), None, None)] == "KLEIN_ERR_ALIGN"
    assert kb.STATUS[kb.lib.klein_positions(ctypes.byref(seq), 4100, None)] == "KLEIN_ERR_ALIGN"
    bad = kb.make_seq(1, 80, 8, 8, ((4, 4),))
    bad.ref_w[0] = 0
    assert kb.STATUS[kb.lib.klein_positions(ctypes.byref(bad), 4096, None)] == "KLEIN_ERR_SHAPE"
    assert kb.lib.klein_stack_workspace_size(ctypes.byref(bad)) == 0


def test_nvfp4_argument_errors_before_any_launch(kb):
    q = kb.lib.klein_quantize_nvfp4
    st = kb.STATUS
    assert st[q(None, 4, 64, 0, 1 << 20, 2 << 20, 3 << 20, None)] == "KLEIN_ERR_INVALID_ARG"
    assert st[q(4104, 4, 64, 0, 1 << 20, 2 << 20, 3 << 20, None)] == "KLEIN_ERR_ALIGN"
    assert st[q(4096, 4, 64, 7, 1 << 20, 2 << 20, 3 << 20, None)] == "KLEIN_ERR_INVALID_ARG"      # mode
    assert st[q(4096, 4, 48, 0, 1 << 20, 2 << 20, 3 << 20, None)] == "KLEIN_ERR_SHAPE"            # cols % 64
    assert st[q(4096, 4, 12352, 0, 1 << 20, 2 << 20, 3 << 20, None)] == "KLEIN_ERR_SHAPE"         # cols > 12288
    assert st[q(4096, 4, 3072, kb.NVFP4_IN_PROJ, 1 << 20, 2 << 20, 3 << 20, None)] == "KLEIN_ERR_SHAPE"
    assert st[q(4096, 4, 64, 0, 4096 + 64, 2 << 20, 3 << 20, None)] == "KLEIN_ERR_INVALID_ARG"    # codes overlap src
    m = kb.lib.klein_op_modln_nvfp4
    assert st[m(None, 1, 10, 0, 10, 5, 5, 4096, 9216, 1 << 20, 2 << 20, 3 << 20, None)] == "KLEIN_ERR_INVALID_ARG"
    assert st[m(4096, 1, 10, 0, 10, 5, 5, 4096, 9214, 1 << 20, 2 << 20, 3 << 20, None)] == "KLEIN_ERR_ALIGN"
    assert st[m(4096, 1, 10, 4, 10, 5, 5, 4096, 9216, 1 << 20, 2 << 20, 3 << 20, None)] == "KLEIN_ERR_SHAPE"
    g = kb.lib.klein_op_gemm_nvfp4
    ptrs = [(k + 1) << 20 for k in range(7)]
    assert st[g(None, *ptrs[1:], 256, 256, 256, None)] == "KLEIN_ERR_INVALID_ARG"
    assert st[g(*ptrs, 256, 200, 256, None)] == "KLEIN_ERR_SHAPE"     # N not a multiple of 128
    assert st[g(*ptrs, 256, 256, 128, None)] == "KLEIN_ERR_SHAPE"     # K not a multiple of 256
    # NVFP4 block weights need both block-scale arrays and both second-level scales
    bw = kb.KleinBlockWeights(16, 32, 48, 64, None, None, 80, 96)
    rc = kb.lib.klein_block_forward(ctypes.byref(bw), 256, 1, 10, 0, 10, 5, 5, 256, 256, 256, 1 << 30, None)
    assert st[rc] == "KLEIN_ERR_INVALID_ARG"
    assert b"second-level scales" in kb.lib.klein_last_error()
    bw = kb.KleinBlockWeights(16, 32, 48, 64, 112, 128, 80, None)
    rc = kb.lib.klein_block_forward(ctypes.byref(bw), 256, 1, 10, 0, 10, 5, 5, 256, 256, 256, 1 << 30, None)
    assert st[rc] == "KLEIN_ERR_INVALID_ARG"
    assert b"w_in_sf and w_out_sf" in kb.lib.klein_last_error()


def test_attention_argument_errors_before_any_launch(kb):
    a = kb.lib.klein_op_attention
    st = kb.STATUS
    p = [(k + 1) << 20 for k in range(4)]
    assert st[a(None, p[1], p[2], 1, 128, 128, p[3], 3072, None)] == "KLEIN_ERR_INVALID_ARG"
    assert st[a(*p[:3], 1, 128, 128, p[3], 3076, None)] == "KLEIN_ERR_ALIGN"          # out_ld % 8
    assert st[a(*p[:3], 1, 128, 120, p[3], 3072, None)] == "KLEIN_ERR_SHAPE"          # rows_pad < rows
    assert st[a(*p[:3], 1, 128, 132, p[3], 3072, None)] == "KLEIN_ERR_SHAPE"          # rows_pad % 8
    assert st[a(*p[:3], 1, 128, 128, p[3], 2048, None)] == "KLEIN_ERR_SHAPE"          # out_ld < 3072
    assert st[a(*p[:3], 0, 128, 128, p[3], 3072, None)] == "KLEIN_ERR_SHAPE"
