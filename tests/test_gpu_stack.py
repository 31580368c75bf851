"""GPU parity of the modulation, the two-stage stack and the Euler sampler
against the oracle, on random-init stacks of reduced depth (the full 5 + 28
stack is compared with stored oracle outputs in test_gpu_full_size.py)."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import klein_inputs as ki  # noqa: E402
import oracle as o  # noqa: E402
from gpu_util import cosine, host, max_err_ratio, to_bf16, to_f32, upload_model, workspace  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kb():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from conftest import ensure_built
    ensure_built()
    import latent_flow_matching_joint_b200 as kb
    return kb


@pytest.fixture(scope="module")
def distilled(kb):
    m = ki.ModelWeights(seed=0, distilled=True, n_stage1=1, n_joint=2)
    t = upload_model(m)
    return m, t, kb.KleinModel(t)


@pytest.fixture(scope="module")
def base(kb):
    m = ki.ModelWeights(seed=0, distilled=False, n_stage1=1, n_joint=1)
    t = upload_model(m, with_ref=False)
    return m, t, kb.KleinModel(t)


@pytest.mark.parametrize("sigma,sigma_next,with_ref", [(0.7, 0.5, True), (1.0, 0.99, False), (0.316, 0.0, True)])
def test_time_modulation(kb, distilled, sigma, sigma_next, with_ref):
    m, _, model = distilled
    mod = torch.zeros((2, 3, 3, ki.DIM), dtype=torch.float32, device="cuda")
    fin = torch.zeros((2, ki.DIM), dtype=torch.float32, device="cuda")
    ws = torch.empty(32768, dtype=torch.float32, device="cuda")
    kb.klein_op_time_mod(model, sigma, sigma_next, with_ref, mod, fin, ws)
    torch.cuda.synchronize()
    ref = o.stage_modulations(m.misc, sigma, sigma_next)
    for st in (1, 2):
        for md in range(3 if with_ref else 2):
            r = ref[st][md]
            g = host(mod[st - 1, md])
            assert np.max(np.abs(g - r)) <= 2e-3 * np.sqrt(np.mean(r * r)), (st, md)
    r = ref["final"]
    assert np.max(np.abs(host(fin) - r)) <= 2e-3 * np.sqrt(np.mean(r * r))


def test_time_modulation_base_model_ignores_target(kb, base):
    m, _, model = base
    mod = torch.zeros((2, 3, 3, ki.DIM), dtype=torch.float32, device="cuda")
    fin = torch.zeros((2, ki.DIM), dtype=torch.float32, device="cuda")
    ws = torch.empty(32768, dtype=torch.float32, device="cuda")
    kb.klein_op_time_mod(model, 0.6, 0.123, False, mod, fin, ws)
    torch.cuda.synchronize()
    ref = o.stage_modulations(m.misc, 0.6, None)
    r = ref[2][1]
    assert np.max(np.abs(host(mod[1, 1]) - r)) <= 2e-3 * np.sqrt(np.mean(r * r))


def _seq_inputs(kb, batch, n_txt, gh, gw, refs, tag):
    seq = kb.make_seq(batch, n_txt, gh, gw, refs)
    n_img, n_ref, n_total = kb.klein_seq_tokens(seq)
    lat = ki.noise_latents(2, n_img)
    text = ki.text_embeddings(1, batch, n_txt)
    rl = ki.ref_latents(1, n_ref) if n_ref else None
    return seq, n_img, n_ref, n_total, lat, text, rl


@pytest.mark.parametrize("n_txt,img,refs", [(80, (8, 8), ((4, 6),)), (37, (5, 9), ()), (80, (8, 8), ())])
def test_stack_forward_matches_oracle(kb, distilled, n_txt, img, refs):
    m, _, model = distilled
    seq, n_img, n_ref, n_total, lat, text, rl = _seq_inputs(kb, 1, n_txt, img[0], img[1], refs, "stack")
    v = torch.full((1, n_img, 128), float("nan"), dtype=torch.float32, device="cuda")
    ws = workspace(kb.klein_stack_workspace_size(seq))
    kb.klein_stack_forward(model, to_f32(lat), to_bf16(text), to_f32(rl) if rl is not None else None, 0.7, 0.5,
                           seq, v, ws)
    torch.cuda.synchronize()
    ref = o.transformer(m, lat, text, rl, o.positions(n_txt, img, refs), 0.7, 0.5)
    got = host(v)
    assert np.all(np.isfinite(got))
    assert cosine(got, ref) >= 0.999, cosine(got, ref)
    assert max_err_ratio(got, ref) <= 5e-2, max_err_ratio(got, ref)


def test_denoise_distilled_with_reference(kb, distilled):
    m, _, model = distilled
    refs = ((4, 4),)
    seq, n_img, n_ref, n_total, lat, text, rl = _seq_inputs(kb, 1, 40, 6, 6, refs, "den")
    x = to_f32(lat)
    x0 = torch.empty_like(x)
    ws = workspace(kb.klein_stack_workspace_size(seq))
    kb.klein_denoise(model, x, to_bf16(text), to_f32(rl), 3, 1.0, seq, ws, x0_out=x0)
    torch.cuda.synchronize()
    last = {}

    def on_step(i, xi, vi, s):
        last["x0"] = o.x0_preview(xi, vi, s)

    ref = o.denoise(m, lat, text, rl, o.positions(40, (6, 6), refs), 3, on_step=on_step)
    assert cosine(host(x), ref) >= 0.999
    assert max_err_ratio(host(x), ref) <= 5e-2
    assert cosine(host(x0), last["x0"]) >= 0.999


def test_denoise_base_cfg(kb, base):
    m, _, model = base
    seq, n_img, n_ref, n_total, lat, text, rl = _seq_inputs(kb, 2, 48, 5, 6, (), "cfg")
    x = to_f32(lat)
    ws = workspace(kb.klein_stack_workspace_size(seq))
    kb.klein_denoise(model, x, to_bf16(text), None, 2, 3.5, seq, ws)
    torch.cuda.synchronize()
    ref = o.denoise(m, lat, text, None, o.positions(48, (5, 6)), 2, cfg=3.5)
    assert cosine(host(x), ref) >= 0.999
    assert max_err_ratio(host(x), ref) <= 5e-2


def test_denoise_argument_errors(kb, base):
    _, _, model = base
    seq, n_img, n_ref, n_total, lat, text, rl = _seq_inputs(kb, 1, 8, 2, 2, (), "err")
    x = to_f32(lat)
    ws = workspace(kb.klein_stack_workspace_size(seq))
    with pytest.raises(kb.KleinError) as e:
        kb.klein_denoise(model, x, to_bf16(text), None, 2, 3.5, seq, ws)   # guidance needs batch 2
    assert e.value.name == "KLEIN_ERR_SHAPE"
    with pytest.raises(kb.KleinError) as e:
        kb.klein_denoise(model, x, to_bf16(text), None, 2, 1.0, seq, ws[:1024])
    assert e.value.name == "KLEIN_ERR_WORKSPACE"
    seq_r = kb.make_seq(1, 8, 2, 2, ((2, 2),))
    with pytest.raises(kb.KleinError) as e:   # the base fixture has no reference weights
        kb.klein_stack_forward(model, x, to_bf16(text), x, 0.5, 0.0, seq_r,
                               torch.empty((1, 4, 128), device="cuda"), workspace(kb.klein_stack_workspace_size(seq_r)))
    assert e.value.name == "KLEIN_ERR_INVALID_ARG"


def test_stack_forward_with_text_projection(kb):
    # text given as the stacked encoder hidden states (8 x 2560 per token),
    # projected to 3072 by the model's txt_in; batch 2 (distinct texts)
    m = ki.ModelWeights(seed=0, distilled=True, n_stage1=1, n_joint=1, txt_in=True)
    t = upload_model(m, with_ref=False)
    model = kb.KleinModel(t)
    n_txt, img = 24, (4, 5)
    seq = kb.make_seq(2, n_txt, img[0], img[1])
    n_img, _, _ = kb.klein_seq_tokens(seq)
    lat = ki.noise_latents(2, n_img)
    hid = ki.text_hidden_states(1, 2, n_txt)
    v = torch.full((2, n_img, 128), float("nan"), dtype=torch.float32, device="cuda")
    ws = workspace(kb.klein_stack_workspace_size(seq))
    kb.klein_stack_forward(model, to_f32(lat), to_bf16(hid), None, 0.6, 0.4, seq, v, ws)
    torch.cuda.synchronize()
    ref = o.transformer(m, lat, hid, None, o.positions(n_txt, img), 0.6, 0.4)
    got = host(v)
    assert np.all(np.isfinite(got))
    assert cosine(got, ref) >= 0.999, cosine(got, ref)
    assert max_err_ratio(got, ref) <= 5e-2, max_err_ratio(got, ref)


def test_denoise_base_with_reference_uses_stage1_cache(kb):
    # base model (no target-level embedder): the text and reference streams'
    # stage-1 output is computed at the first step and reused; the result
    # must still match the oracle, which recomputes everything every step
    m = ki.ModelWeights(seed=3, distilled=False, n_stage1=2, n_joint=1)
    t = upload_model(m)
    model = kb.KleinModel(t)
    refs = ((3, 4),)
    seq, n_img, n_ref, n_total, lat, text, rl = _seq_inputs(kb, 2, 20, 5, 4, refs, "cache")
    x = to_f32(lat)
    ws = workspace(kb.klein_stack_workspace_size(seq))
    kb.klein_denoise(model, x, to_bf16(text), to_f32(rl), 3, 2.0, seq, ws)
    torch.cuda.synchronize()
    ref = o.denoise(m, lat, text, rl, o.positions(20, (5, 4), refs), 3, cfg=2.0)
    assert cosine(host(x), ref) >= 0.999
    assert max_err_ratio(host(x), ref) <= 5e-2


@pytest.fixture(scope="module")
def distilled_refs(kb):
    m = ki.ModelWeights(seed=5, distilled=True, n_stage1=1, n_joint=2)
    t = upload_model(m)
    return m, t, kb.KleinModel(t)


THREE_REFS = ((4, 6), (3, 5), (6, 2))   # three reference images, each its own grid size


def test_stack_forward_three_references(kb, distilled_refs):
    # an edit with three references of different sizes: each takes its own l
    # offset (-1, -2, -3) and all join the reference stream of stage 1
    m, _, model = distilled_refs
    seq, n_img, n_ref, n_total, lat, text, rl = _seq_inputs(kb, 1, 48, 5, 7, THREE_REFS, "refs3")
    assert n_ref == 24 + 15 + 12
    v = torch.full((1, n_img, 128), float("nan"), dtype=torch.float32, device="cuda")
    ws = workspace(kb.klein_stack_workspace_size(seq))
    kb.klein_stack_forward(model, to_f32(lat), to_bf16(text), to_f32(rl), 0.8, 0.6, seq, v, ws)
    torch.cuda.synchronize()
    ref = o.transformer(m, lat, text, rl, o.positions(48, (5, 7), THREE_REFS), 0.8, 0.6)
    got = host(v)
    assert np.all(np.isfinite(got))
    assert cosine(got, ref) >= 0.999, cosine(got, ref)
    assert max_err_ratio(got, ref) <= 5e-2, max_err_ratio(got, ref)


def test_denoise_three_references(kb, distilled_refs):
    m, _, model = distilled_refs
    seq, n_img, n_ref, n_total, lat, text, rl = _seq_inputs(kb, 1, 32, 4, 6, THREE_REFS, "refs3den")
    x = to_f32(lat)
    ws = workspace(kb.klein_stack_workspace_size(seq))
    kb.klein_denoise(model, x, to_bf16(text), to_f32(rl), 3, 1.0, seq, ws)
    torch.cuda.synchronize()
    ref = o.denoise(m, lat, text, rl, o.positions(32, (4, 6), THREE_REFS), 3)
    assert cosine(host(x), ref) >= 0.999
    assert max_err_ratio(host(x), ref) <= 5e-2


def test_denoise_x0_preview_every_step(kb, distilled):
    # the x0 preview x - sigma v of every step (before its update), as the
    # pages' preview block shows after each denoiser call
    m, _, model = distilled
    seq, n_img, n_ref, n_total, lat, text, rl = _seq_inputs(kb, 1, 40, 6, 6, (), "x0steps")
    steps = 3
    x = to_f32(lat)
    x0 = torch.full((steps, n_img, 128), float("nan"), dtype=torch.float32, device="cuda")
    ws = workspace(kb.klein_stack_workspace_size(seq))
    kb.klein_denoise(model, x, to_bf16(text), None, steps, 1.0, seq, ws, x0_out=x0, x0_every_step=True)
    torch.cuda.synchronize()
    previews = {}

    def on_step(i, xi, vi, s):
        previews[i] = o.x0_preview(xi, vi, s)

    ref = o.denoise(m, lat, text, None, o.positions(40, (6, 6)), steps, on_step=on_step)
    assert cosine(host(x), ref) >= 0.999
    got = host(x0)
    for i in range(steps):
        assert np.all(np.isfinite(got[i])), i
        assert cosine(got[i], previews[i]) >= 0.999, (i, cosine(got[i], previews[i]))
        assert max_err_ratio(got[i], previews[i]) <= 5e-2, (i, max_err_ratio(got[i], previews[i]))
