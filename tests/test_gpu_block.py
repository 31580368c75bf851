"""GPU parity of klein_block_forward against the oracle block.

Tolerance (per block): max |GPU - oracle| <= 2e-2 * RMS(oracle block output).
The block delta (gate * (attention + MLP)) is also checked, with a looser
bound, because the residual x dominates the output RMS."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import klein_inputs as ki  # noqa: E402
import oracle as o  # noqa: E402
from gpu_util import cosine, host, max_err_ratio, to_f32, upload_block, workspace  # noqa: E402

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
def weights():
    w = ki.block_weights(0, "joint.0")
    return w, upload_block(w)


def run_block(kb, wd, x, seq, mod, row0, rows, n_txt, n_img):
    batch, n_total = x.shape[0], x.shape[1]
    xd = to_f32(x)
    pos = torch.empty((n_total, 4), dtype=torch.float32, device="cuda")
    kb.klein_positions(seq, pos)
    ws = workspace(kb.klein_block_workspace_size(batch, rows))
    kb.klein_block_forward(wd, xd, n_txt, n_img, pos, to_f32(mod), ws, row0=row0, rows=rows)
    torch.cuda.synchronize()
    return host(xd)


CASES = {
    # config 1: 80 text tokens + 8x8 image, batch 1
    "config1": dict(batch=1, n_txt=80, img=(8, 8), refs=(), view="joint"),
    # ragged: 155 rows (not a multiple of 128), with a reference, batch 2
    "ragged_ref_b2": dict(batch=2, n_txt=77, img=(9, 7), refs=((3, 5),), view="joint"),
    # stage-1 image stream: rows [n_txt, n_txt + n_img) attend only to themselves
    "stage1_image": dict(batch=1, n_txt=80, img=(12, 11), refs=(), view="img"),
    "stage1_text_b2": dict(batch=2, n_txt=150, img=(4, 4), refs=(), view="txt"),
    "tiny": dict(batch=1, n_txt=1, img=(1, 1), refs=(), view="joint"),
}


@pytest.mark.parametrize("name", list(CASES))
def test_block_matches_oracle(kb, weights, name):
    c = CASES[name]
    w, wd = weights
    n_txt, (gh, gw), refs = c["n_txt"], c["img"], c["refs"]
    n_img = gh * gw
    n_ref = sum(h * ww for h, ww in refs)
    n_total = n_txt + n_img + n_ref
    seq = kb.make_seq(c["batch"], n_txt, gh, gw, refs)
    x = ki.tokens(1, f"block.{name}", c["batch"], n_total)
    mod = ki.modulation_vectors(1, f"block.{name}")
    row0, rows = {"joint": (0, n_total), "img": (n_txt, n_img), "txt": (0, n_txt)}[c["view"]]
    got = run_block(kb, wd, x, seq, mod, row0, rows, n_txt, n_img)

    pos = o.positions(n_txt, (gh, gw), refs)
    modes = o.mode_of_rows(n_txt, n_img, n_ref)
    sl = slice(row0, row0 + rows)
    ref = o.block(x[:, sl], pos[sl], modes[sl], mod.astype(np.float64), w)
    # rows outside the view are untouched
    mask = np.ones(n_total, bool)
    mask[sl] = False
    np.testing.assert_array_equal(got[:, mask], x[:, mask])
    g = got[:, sl]
    assert np.all(np.isfinite(g))
    assert max_err_ratio(g, ref) <= 2e-2, max_err_ratio(g, ref)
    d_ref = ref - x[:, sl]
    d_got = g - x[:, sl]
    assert cosine(d_got, d_ref) >= 0.999
    assert max_err_ratio(d_got, d_ref) <= 0.1


@pytest.mark.parametrize("batch,n_txt,grid,refs", [
    (1, 512, (64, 64), ((64, 64),)),     # 1024x1024 edit: 512 + 4096 + 4096 = 8704 tokens
    (2, 560, (128, 128), ()),            # 2048x2048 base with guidance: 2 x (560 + 16384) = 2 x 16944
    (1, 512, (256, 256), ()),            # the largest output, 4096x4096: 512 + 65536 tokens
    (3, 160, (16, 16), ((8, 8), (4, 6))),  # batch 3, two references
])
def test_block_large_sampled_rows(kb, weights, batch, n_txt, grid, refs):
    # full-size joint blocks of the edit and 2048x2048 workloads; the oracle
    # evaluates a sample of output rows (every row supplies keys and values)
    w, wd = weights
    n_img = grid[0] * grid[1]
    n_ref = sum(h * ww for h, ww in refs)
    n_total = n_txt + n_img + n_ref
    seq = kb.make_seq(batch, n_txt, grid[0], grid[1], refs)
    x = ki.tokens(1, f"block.large.{n_total}", batch, n_total)
    mod = ki.modulation_vectors(1, f"block.large.{n_total}")
    got = run_block(kb, wd, x, seq, mod, 0, n_total, n_txt, n_img)
    rows = np.unique(np.concatenate([np.arange(0, n_total, 997), [0, n_txt - 1, n_txt, n_txt + n_img,
                                                                 n_total - 1]]))
    rows = rows[rows < n_total]
    ref = o.block(x, o.positions(n_txt, grid, refs), o.mode_of_rows(n_txt, n_img, n_ref),
                  mod.astype(np.float64), w, rows=rows)
    g = got[:, rows]
    assert np.all(np.isfinite(g))
    assert max_err_ratio(g, ref) <= 2e-2, max_err_ratio(g, ref)
    assert cosine(g - x[:, rows], ref - x[:, rows]) >= 0.999


def test_block_config2_sampled_rows(kb, weights):
    # 1024x1024 text-to-image joint block: 512 text + 64x64 image, batch 1;
    # the oracle computes a sample of output rows (all rows give keys/values).
    w, wd = weights
    n_txt, gh, gw = 512, 64, 64
    n_total = n_txt + gh * gw
    seq = kb.make_seq(1, n_txt, gh, gw)
    x = ki.tokens(1, "block.config2", 1, n_total)
    mod = ki.modulation_vectors(1, "block.config2")
    got = run_block(kb, wd, x, seq, mod, 0, n_total, n_txt, gh * gw)
    rows = np.unique(np.concatenate([np.arange(0, n_total, 151), [0, 511, 512, 4607, 4606]]))
    ref = o.block(x, o.positions(n_txt, (gh, gw)), o.mode_of_rows(n_txt, gh * gw, 0), mod.astype(np.float64), w,
                  rows=rows)
    g = got[:, rows]
    assert max_err_ratio(g, ref) <= 2e-2
    assert cosine(g - x[:, rows], ref - x[:, rows]) >= 0.999
