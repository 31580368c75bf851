"""GPU parity at the full model depth (5 + 28 blocks) against stored oracle
outputs: the 16-step distilled denoise of 80 text + 8x8 image tokens, one
denoiser call at the benchmarked 1024x1024 text-to-image size (512 text +
64x64 image tokens) and at the 1024x1024 edit size (+ one 64x64 reference),
and the full 16-step denoise at 512 + 64x64 tokens.

The stored files are written by tests/golden/make_denoise_golden.py and
tests/golden/make_full_size_goldens.py, which call only the oracle and the
seeded input generators. The benchmark spec's bounds: cosine >= 0.999 of the
velocities and the final latents; max |GPU - oracle| <= 5e-2 x RMS(oracle) is
an additional bound of this repository (the per-block 2e-2 x RMS compounded
over 33 blocks of bf16 storage, measured at 1.7-3.1e-2 on the reduced
stacks)."""
import json
import os

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import klein_inputs as ki  # noqa: E402
from gpu_util import cosine, host, max_err_ratio, to_bf16, to_f32, upload_model, workspace  # noqa: E402

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


@pytest.fixture(scope="module")
def kb():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from conftest import ensure_built
    ensure_built()
    import latent_flow_matching_joint_b200 as kb
    return kb


@pytest.fixture(scope="module")
def full_model(kb):
    """The random-init 5 + 28 block distilled stack on the device (about
    10.5 GB of bf16 weights), generated once for this module."""
    m = ki.ModelWeights(seed=ki.WEIGHT_SEED, distilled=True)
    t = upload_model(m)
    m._blocks.clear()     # the host copies are not needed after the upload
    return t, kb.KleinModel(t)


def _golden(name):
    path = os.path.join(GOLDEN, name + ".npy")
    with open(path.replace(".npy", ".json")) as f:
        meta = json.load(f)
    return np.load(path).astype(np.float64), meta


def _inputs(kb, meta):
    n_txt, (gh, gw) = meta["n_txt"], meta["grid"]
    refs = tuple(tuple(r) for r in meta.get("refs", ()))
    seq = kb.make_seq(1, n_txt, gh, gw, refs)
    n_img, n_ref, _ = kb.klein_seq_tokens(seq)
    lat = to_f32(ki.noise_latents(meta["noise_seed"], n_img))
    text = to_bf16(ki.text_embeddings(meta["text_seed"], 1, n_txt))
    rl = to_f32(ki.ref_latents(meta["ref_seed"], n_ref)) if n_ref else None
    return seq, n_img, lat, text, rl


def _check(got, ref):
    assert np.all(np.isfinite(got))
    assert cosine(got, ref) >= 0.999, cosine(got, ref)
    assert max_err_ratio(got, ref) <= 5e-2, max_err_ratio(got, ref)


def test_full_depth_denoise_80_8x8(kb, full_model):
    ref, meta = _golden("denoise_full_depth_80_8x8_16")
    meta.setdefault("ref_seed", ki.INPUT_SEED)
    _, model = full_model
    seq, n_img, x, text, _ = _inputs(kb, meta)
    ws = workspace(kb.klein_stack_workspace_size(seq))
    kb.klein_denoise(model, x, text, None, meta["steps"], 1.0, seq, ws)
    torch.cuda.synchronize()
    _check(host(x), ref)


@pytest.mark.parametrize("name", ["stack_t2i_1024", "stack_edit_1024"])
def test_full_size_stack_velocity(kb, full_model, name):
    ref, meta = _golden(name)
    _, model = full_model
    seq, n_img, lat, text, rl = _inputs(kb, meta)
    v = torch.full((1, n_img, 128), float("nan"), dtype=torch.float32, device="cuda")
    ws = workspace(kb.klein_stack_workspace_size(seq))
    kb.klein_stack_forward(model, lat, text, rl, meta["sigma"], meta["sigma_next"], seq, v, ws)
    torch.cuda.synchronize()
    _check(host(v), ref)
    assert kb.klein_device_status()[0] == 0


def test_full_size_denoise_t2i_1024(kb, full_model):
    # the benchmarked workload: 16 shifted Euler steps at 512 + 64x64 tokens
    ref, meta = _golden("denoise_t2i_1024")
    _, model = full_model
    seq, n_img, x, text, _ = _inputs(kb, meta)
    ws = workspace(kb.klein_stack_workspace_size(seq))
    kb.klein_denoise(model, x, text, None, meta["steps"], 1.0, seq, ws)
    torch.cuda.synchronize()
    _check(host(x), ref)
    assert kb.klein_device_status()[0] == 0


def test_stack_t2i4k_sampled_rows(kb):
    # the largest output, 4096x4096 (512 text + 256x256 image tokens): a
    # 0 + 1 block stack (the model's first joint block) through
    # klein_stack_forward, against the oracle's velocity on a sample of
    # image rows
    ref, meta = _golden("stack_t2i4k_rows")
    m = ki.ModelWeights(seed=meta["weight_seed"], distilled=True, n_stage1=0, n_joint=1)
    t = upload_model(m, with_ref=False)
    model = kb.KleinModel(t)
    seq, n_img, lat, text, rl = _inputs(kb, meta)
    v = torch.full((1, n_img, 128), float("nan"), dtype=torch.float32, device="cuda")
    ws = workspace(kb.klein_stack_workspace_size(seq))
    kb.klein_stack_forward(model, lat, text, rl, meta["sigma"], meta["sigma_next"], seq, v, ws)
    torch.cuda.synchronize()
    got = host(v)
    assert np.all(np.isfinite(got))
    _check(got[:, np.asarray(meta["img_rows"])], ref)
    assert kb.klein_device_status()[0] == 0
