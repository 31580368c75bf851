"""GPU parity of the single kernels against the oracle (float64 CPU)."""
import math

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import klein_inputs as ki  # noqa: E402
import oracle as o  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kb():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from conftest import ensure_built
    ensure_built()
    import latent_flow_matching_joint_b200 as kb
    return kb


from gpu_util import cosine, host, rms, to_bf16, to_f32  # noqa: E402


# ------------------------------------------------------------------ GEMM

@pytest.mark.parametrize("m,n,k", [(128, 256, 64), (300, 384, 192), (1, 128, 64), (1000, 512, 3072),
                                   (777, 3072, 128), (4608, 256, 12288)])
def test_gemm_matches_fp64(kb, m, n, k):
    a = ki.normal(11, f"gemm.a.{m}.{n}.{k}", (m, k))
    b = ki.normal(11, f"gemm.b.{m}.{n}.{k}", (n, k), std=1 / math.sqrt(k))
    c = torch.full((m, n), float("nan"), dtype=torch.float32, device="cuda")
    kb.klein_op_gemm(to_bf16(a), to_bf16(b), c)
    torch.cuda.synchronize()
    ref = a.astype(np.float64) @ b.astype(np.float64).T
    got = host(c)
    assert np.all(np.isfinite(got))
    # fp32 accumulation of exact bf16 products: relative error ~ 1e-6
    assert np.max(np.abs(got - ref)) <= 1e-4 * rms(ref) + 1e-6


# ------------------------------------------------------------------ modLN

@pytest.mark.parametrize("batch,n_txt,n_img,n_ref,row0,rows", [
    (1, 80, 64, 0, 0, 144), (2, 77, 63, 15, 0, 155), (1, 512, 4096, 0, 0, 4608), (2, 30, 20, 10, 30, 20)])
def test_modln(kb, batch, n_txt, n_img, n_ref, row0, rows):
    n_total = n_txt + n_img + n_ref
    x = ki.tokens(1, f"modln.{n_total}", batch, n_total)
    mod = ki.modulation_vectors(1, f"modln.{n_total}")
    h = torch.empty((batch, rows, ki.DIM), dtype=torch.bfloat16, device="cuda")
    kb.klein_op_modln(to_f32(x), row0, rows, n_txt, n_img, to_f32(mod), h)
    torch.cuda.synchronize()
    modes = o.mode_of_rows(n_txt, n_img, n_ref)
    ref = o.modln(x, modes, mod.astype(np.float64))[:, row0:row0 + rows]
    got = host(h)
    # one bf16 rounding of each output
    assert np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-5)


def test_modln_context_rows_ignore_image_modulation(kb):
    # text rows of h are bit-identical whatever the image (mode 1) modulation is
    x = to_f32(ki.tokens(1, "modln.ctx", 1, 40))
    mod = ki.modulation_vectors(1, "modln.ctx")
    mod2 = mod.copy()
    mod2[1] *= 3.0
    h1 = torch.empty((1, 40, ki.DIM), dtype=torch.bfloat16, device="cuda")
    h2 = torch.empty_like(h1)
    kb.klein_op_modln(x, 0, 40, 16, 24, to_f32(mod), h1)
    kb.klein_op_modln(x, 0, 40, 16, 24, to_f32(mod2), h2)
    torch.cuda.synchronize()
    assert torch.equal(h1[:, :16], h2[:, :16])
    assert not torch.equal(h1[:, 16:], h2[:, 16:])


# ------------------------------------------------------------------ positions + RoPE

@pytest.mark.parametrize("n_txt,img,refs", [(80, (8, 8), ()), (512, (64, 64), ((64, 64),)),
                                            (7, (3, 5), ((2, 2), (1, 3), (4, 1)))])
def test_positions(kb, n_txt, img, refs):
    seq = kb.make_seq(1, n_txt, img[0], img[1], refs)
    _, _, nt = kb.klein_seq_tokens(seq)
    pos = torch.empty((nt, 4), dtype=torch.float32, device="cuda")
    kb.klein_positions(seq, pos)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host(pos), o.positions(n_txt, img, refs))


@pytest.mark.parametrize("n_txt,img,refs,heads", [(80, (8, 8), (), 24), (512, (64, 64), ((64, 64),), 2),
                                                  (13, (5, 7), ((3, 3),), 3)])
def test_rope(kb, n_txt, img, refs, heads):
    seq = kb.make_seq(1, n_txt, img[0], img[1], refs)
    _, _, nt = kb.klein_seq_tokens(seq)
    pos = torch.empty((nt, 4), dtype=torch.float32, device="cuda")
    kb.klein_positions(seq, pos)
    table = torch.empty((nt, 64, 2), dtype=torch.float32, device="cuda")
    kb.klein_op_rope_table(pos, table)
    x = ki.normal(3, f"rope.{nt}.{heads}", (nt, heads, 128))
    out = torch.empty((nt, heads, 128), dtype=torch.bfloat16, device="cuda")
    kb.klein_op_rope(to_bf16(x), out, table)
    torch.cuda.synchronize()
    ref = o.rope(x, o.positions(n_txt, img, refs))
    got = host(out)
    assert np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 2e-6 * np.abs(x).max())


# ------------------------------------------------------------------ Euler / CFG

@pytest.mark.parametrize("guided", [False, True])
def test_euler(kb, guided):
    n_img = 4096
    x = ki.noise_latents(2, n_img)
    v = ki.velocity(5, "euler", 2, n_img)
    xt = to_f32(x)
    x0 = torch.empty_like(xt)
    vc, vu = to_f32(v[0]), to_f32(v[1])
    sig, sig_n, g = 0.615, 0.497, 3.5
    kb.klein_op_euler(xt, vc, vu if guided else None, sig_n - sig, g, x0_out=x0, sigma=sig)
    torch.cuda.synchronize()
    vv = o.cfg_combine(v[0], v[1], g) if guided else v[0].astype(np.float64)
    ref = o.euler_step(x, vv, sig, sig_n)
    ref0 = o.x0_preview(x, vv, sig)
    np.testing.assert_allclose(host(xt), ref, rtol=1e-5, atol=1e-5)
    np.testing.assert_allclose(host(x0), ref0, rtol=1e-5, atol=1e-5)


# ------------------------------------------------------------------ attention

def _attn_inputs(batch, rows, heads_used, tag):
    rp = (rows + 127) // 128 * 128
    q = ki.normal(7, f"attn.q.{tag}", (batch, rows, 24, 128))
    k = ki.normal(7, f"attn.k.{tag}", (batch, rows, 24, 128))
    v = ki.normal(7, f"attn.v.{tag}", (batch, rows, 24, 128))
    qd = torch.zeros((batch, 24, rp, 128), dtype=torch.bfloat16, device="cuda")
    kd = torch.zeros_like(qd)
    vtd = torch.full((batch, 24, 128, rp), float("nan"), dtype=torch.bfloat16, device="cuda")
    qd[:, :, :rows] = to_bf16(q).permute(0, 2, 1, 3)
    kd[:, :, :rows] = to_bf16(k).permute(0, 2, 1, 3)
    vtd[:, :, :, :rows] = to_bf16(v).permute(0, 2, 3, 1)
    return q, k, v, qd, kd, vtd


def attention_bound(q, k, v, ref):
    """Elementwise error bound of the kernel's arithmetic: the output is
    rounded once to bf16 (<= 2^-9 |o|) and the probabilities are rounded to
    bf16 before the P.V product (<= 2^-9 sum_j p_j |v_j| / l, i.e. 2^-9 times
    attention applied to |v|); both doubled for the approximate exp2 and the
    fp32 accumulation order."""
    return 2.0 ** -8 * (np.abs(ref) + o.attention(q, k, np.abs(v))) + 1e-6


@pytest.mark.parametrize("batch,rows", [(1, 144), (2, 300), (1, 1), (1, 128), (1, 129), (1, 513), (2, 700)])
def test_attention_matches_oracle(kb, batch, rows):
    q, k, v, qd, kd, vtd = _attn_inputs(batch, rows, 24, f"{batch}.{rows}")
    out = torch.full((batch, rows, ki.DIM + ki.MLP_HIDDEN), float("nan"), dtype=torch.bfloat16, device="cuda")
    kb.klein_op_attention(qd, kd, vtd, rows, out)
    torch.cuda.synchronize()
    got = host(out[:, :, :ki.DIM]).reshape(batch, rows, 24, 128)
    ref = o.attention(q, k, v)
    assert np.all(np.isfinite(got))
    assert np.all(np.abs(got - ref) <= attention_bound(q, k, v, ref))
    assert cosine(got, ref) >= 0.9999
    # columns past the attention output are untouched
    assert torch.isnan(out[:, :, ki.DIM:]).all()


@pytest.mark.parametrize("batch,rows", [(1, 200), (2, 700)])
def test_attention_rescales_mid_tile(kb, batch, rows):
    """Scores that climb along the keys: q . k_j grows by about 2 per key, so
    a row's maximum (in exp2 units) rises by ~16 every 64 keys, far past
    the kernel's lazy-rescale threshold of 8, and the running maximum moves
    (and O is rescaled) in every key tile, the last one included. The
    per-row factor s_i in [0, 1.5] leaves some rows of each warp below the
    threshold, so rows that rescale and rows that do not share a warp."""
    rp = (rows + 127) // 128 * 128
    s_i = np.linspace(0.0, 1.5, rows)[None, :, None, None]
    ramp = (np.arange(rows) / 64.0)[None, :, None, None]
    q = ki.round_to_bf16(s_i * (1.0 + 0.1 * ki.normal(8, f"attn.rq.{rows}", (batch, rows, 24, 128))))
    k = ki.round_to_bf16(ramp * (1.0 + 0.1 * ki.normal(8, f"attn.rk.{rows}", (batch, rows, 24, 128))))
    v = ki.normal(8, f"attn.rv.{rows}", (batch, rows, 24, 128))
    qd = torch.zeros((batch, 24, rp, 128), dtype=torch.bfloat16, device="cuda")
    kd = torch.zeros_like(qd)
    vtd = torch.zeros((batch, 24, 128, rp), dtype=torch.bfloat16, device="cuda")
    qd[:, :, :rows] = to_bf16(q).permute(0, 2, 1, 3)
    kd[:, :, :rows] = to_bf16(k).permute(0, 2, 1, 3)
    vtd[:, :, :, :rows] = to_bf16(v).permute(0, 2, 3, 1)
    out = torch.empty((batch, rows, ki.DIM), dtype=torch.bfloat16, device="cuda")
    kb.klein_op_attention(qd, kd, vtd, rows, out)
    torch.cuda.synchronize()
    got = host(out).reshape(batch, rows, 24, 128)
    ref = o.attention(q, k, v)
    assert np.all(np.isfinite(got))
    assert np.all(np.abs(got - ref) <= attention_bound(q, k, v, ref))
    assert cosine(got, ref) >= 0.9999


def test_attention_long_sampled(kb):
    rows = 4608
    q, k, v, qd, kd, vtd = _attn_inputs(1, rows, 24, "long")
    out = torch.empty((1, rows, ki.DIM), dtype=torch.bfloat16, device="cuda")
    kb.klein_op_attention(qd, kd, vtd, rows, out)
    torch.cuda.synchronize()
    sample = np.unique(np.concatenate([np.arange(0, rows, 97), [rows - 1, rows - 2, 511, 512]]))
    got = host(out)[0, sample].reshape(len(sample), 24, 128)
    ref = o.attention(q[:, sample], k, v)[0]
    assert np.all(np.abs(got - ref) <= attention_bound(q[:, sample], k, v, ref[None])[0])
    assert cosine(got, ref) >= 0.9999


# ------------------------------------------------------------------ wait bound

def test_wait_probe_reports_timeout(kb):
    rc, _, _ = kb.klein_device_status()
    assert rc == 0
    kb.klein_wait_probe(2_000_000)  # 2 ms, nothing ever arrives
    rc, site, msg = kb.klein_device_status()
    assert kb.STATUS[rc] == "KLEIN_ERR_TIMEOUT" and site == 0x900, msg
    # the context stays usable and the word is cleared
    a = torch.ones(4, device="cuda")
    assert float(a.sum()) == 4.0
    assert kb.klein_device_status()[0] == 0


def test_sync_reports_timeout_on_its_stream(kb):
    s = torch.cuda.Stream()
    assert kb.klein_sync(s.cuda_stream)[0] == 0
    with torch.cuda.stream(s):
        kb.klein_wait_probe(2_000_000, s.cuda_stream)  # 2 ms, nothing ever arrives
    rc, msg = kb.klein_sync(s.cuda_stream)
    assert kb.STATUS[rc] == "KLEIN_ERR_TIMEOUT", msg
    assert kb.klein_sync(s.cuda_stream)[0] == 0     # read and cleared
    assert kb.klein_device_status()[0] == 0
