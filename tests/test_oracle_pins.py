"""Pins of the CPU oracle to facts outside itself (pages' printed values,
closed forms, invariants, library routines). CPU only."""
import math

import numpy as np
import pytest
import torch

import klein_inputs as ki
import oracle as o


# ---------------------------------------------------------------- schedule

def test_schedule_16_printed_values(golden):
    g = golden("schedule_16.txt")
    s = o.sigma_schedule(16)
    assert len(s) == 17 and s[-1] == 0.0
    np.testing.assert_allclose(np.round(s[:3], 3), g["first"], atol=0)
    np.testing.assert_allclose(np.round(s[13:16], 3), g["last"], atol=0)
    assert round(s[0] - s[1], 3) == g["first_step"]
    assert round(s[15] - s[16], 3) == g["last_step"]
    assert int((s[:-1] > 0.5).sum()) == g["above_half"]


def test_schedule_other_printed_values(golden):
    g = golden("schedule_other.txt")
    s50 = o.sigma_schedule(50, g["shift"])
    assert int((s50[:-1] > 0.5).sum()) == g["steps50_above_half"]
    # "step 10": both 0-based and 1-based readings round to 0.97
    assert round(s50[9], 2) == g["steps50_step10"]
    assert round(s50[10], 2) == g["steps50_step10"]
    s4 = o.sigma_schedule(4)
    assert round(s4[3], 3) == g["steps4_last"] and s4[4] == 0.0


def test_schedule_shift_one_is_linear():
    # shift 1 leaves the evenly spaced levels unchanged (closed form)
    np.testing.assert_allclose(o.sigma_schedule(8, 1.0)[:-1], np.linspace(1, 1 / 8, 8), rtol=0, atol=1e-15)


def test_timesteps_scale():
    np.testing.assert_allclose(o.timesteps([1.0, 0.5, 0.0]), [1000.0, 500.0, 0.0])


# ------------------------------------------------------------- geometry

def test_token_counts(golden):
    g = golden("structure.txt")
    assert o.image_tokens(1024, 1024) == g["tokens_1024x1024"]
    assert o.image_tokens(4096, 4096) == g["tokens_4096x4096"]
    assert o.image_tokens(1024, 1024) == g["ref_tokens_1024x1024"]
    assert o.image_tokens(128, 128) == 64
    assert o.image_tokens(2048, 2048) == 16384
    assert 512 + 2 * o.image_tokens(1024, 1024) == 8704


def test_text_padding(golden):
    g = golden("structure.txt")
    assert o.TEXT_PAD == g["text_pad"]
    assert [o.pad_text_len(n) for n in (1, 79, 80, 81, 160, 512)] == [80, 80, 80, 160, 160, 560]
    assert 8 * 2560 == g["text_stack_dim"]


def test_positions_table():
    p = o.positions(3, (2, 2), refs=((1, 2), (1, 1)))
    expect = [(0, 0, 0, 0), (0, 0, 0, 1), (0, 0, 0, 2),
              (0, 0, 0, 0), (0, 0, 1, 0), (0, 1, 0, 0), (0, 1, 1, 0),
              (0, 0, 0, -1), (0, 0, 1, -1), (0, 0, 0, -2)]
    np.testing.assert_array_equal(p, np.array(expect, float))


def test_parameter_counts(golden):
    g = golden("structure.txt")
    assert o.parameter_count(False) == g["base_params"]
    assert o.parameter_count(True) == g["distilled_params"]
    assert o.parameter_count(True) - o.parameter_count(False) == g["param_diff"]
    assert (o.DIM, o.HEADS, o.HEAD_DIM) == (g["dim"], g["heads"], g["head_dim"])
    assert (o.N_STAGE1, o.N_JOINT, o.AXIS_DIM) == (g["stage1_blocks"], g["joint_blocks"], g["rope_axis_dims"])


def test_generated_weights_match_parameter_layout():
    # The generator's tensors, counted, equal the oracle's structural count
    # (which is pinned to the printed totals) for a 1+1-block stack.
    m = ki.ModelWeights(seed=0, distilled=True, n_stage1=1, n_joint=1)
    n = sum(a.size for a in m.misc.values())
    for mode in ki.MODES:
        n += sum(a.size for a in m.stage1(mode)[0].values())
    n += sum(a.size for a in m.joint()[0].values())
    assert n == o.parameter_count(True, 1, 1, txt_in=False)
    # with the 20480 -> 3072 text input projection
    mt = ki.ModelWeights(seed=0, distilled=False, n_stage1=1, n_joint=1, txt_in=True)
    n_t = sum(a.size for a in mt.misc.values())
    assert n_t - sum(a.size for a in ki.misc_weights(0, False).values()) == 8 * 2560 * o.DIM
    assert o.parameter_count(False, 1, 1, txt_in=True) - o.parameter_count(False, 1, 1, txt_in=False) == 8 * 2560 * o.DIM


def test_text_projection_shapes(golden):
    # eight 2560-wide encoder layers stack to the printed 20480, projected to the width
    g = golden("structure.txt")
    m = ki.ModelWeights(seed=0, distilled=False, n_stage1=1, n_joint=1, txt_in=True)
    assert m.misc["txt_in"].shape == (g["dim"], g["text_stack_dim"])
    assert ki.text_hidden_states(1, 2, 3).shape == (2, 3, g["text_stack_dim"])


# ------------------------------------------------------- embeddings

def test_sinusoid_zero_and_period():
    e = o.timestep_sinusoid(0.0)
    np.testing.assert_array_equal(e[:128], 1.0)
    np.testing.assert_array_equal(e[128:], 0.0)
    # frequency 0 is 1 rad per unit of t: cos/sin of t itself
    e = o.timestep_sinusoid(0.5)
    assert e[0] == pytest.approx(math.cos(0.5)) and e[128] == pytest.approx(math.sin(0.5))
    np.testing.assert_allclose(e[:128] ** 2 + e[128:] ** 2, 1.0, atol=1e-14)


def test_silu_closed_form():
    assert o.silu(0.0) == 0.0
    assert o.silu(1.0) == pytest.approx(1 / (1 + math.exp(-1)))
    assert o.silu(-50.0) == pytest.approx(0.0, abs=1e-18)


def test_context_modes_ignore_image_time():
    m = ki.ModelWeights(seed=0, distilled=False, n_stage1=1, n_joint=1)
    a = o.stage_modulations(m.misc, 0.9, None)
    b = o.stage_modulations(m.misc, 0.2, None)
    for st in (1, 2):
        np.testing.assert_array_equal(a[st][o.MODE_TXT], b[st][o.MODE_TXT])
        np.testing.assert_array_equal(a[st][o.MODE_REF], b[st][o.MODE_REF])
        assert not np.allclose(a[st][o.MODE_IMG], b[st][o.MODE_IMG])
    # image at sigma 0 has the same embedding as the context streams
    c = o.stage_modulations(m.misc, 0.0, None)
    np.testing.assert_array_equal(c[1][o.MODE_IMG], o.modulation(m.misc["mod1.img"], o.time_embedding(m.misc, 0.0, None), 3))


def test_target_embedder_adds_to_every_mode():
    m = ki.ModelWeights(seed=0, distilled=True, n_stage1=1, n_joint=1)
    e1 = o.time_embedding(m.misc, 0.5, 0.3)
    e0 = o.time_embedding(m.misc, 0.5, None)
    e_t = o.time_embed_mlp(m.misc["tt_mlp1"], m.misc["tt_mlp2"], 0.3)
    np.testing.assert_allclose(e1, e0 + e_t, rtol=0, atol=1e-12)
    # context streams at t=0 still see the target embedding
    ctx = o.time_embedding(m.misc, 0.0, 0.3)
    assert not np.allclose(ctx, o.time_embedding(m.misc, 0.0, None))


# ------------------------------------------------------------ norms

def test_layer_norm_moments():
    x = np.random.default_rng(3).normal(2.0, 5.0, size=(7, o.DIM))
    y = o.layer_norm(x)
    np.testing.assert_allclose(y.mean(-1), 0.0, atol=1e-12)
    np.testing.assert_allclose(y.var(-1), 1.0, rtol=1e-6)
    # shift/scale invariance of a no-affine LayerNorm
    np.testing.assert_allclose(o.layer_norm(3 * x + 7), y, atol=1e-9)


def test_modln_modes():
    rng = np.random.default_rng(4)
    x = rng.normal(size=(1, 5, o.DIM))
    mod = rng.normal(size=(3, 3, o.DIM))
    modes = np.array([0, 0, 1, 2, 2])
    h = o.modln(x, modes, mod)
    xh = o.layer_norm(x)
    for r, m in enumerate(modes):
        np.testing.assert_allclose(h[0, r], (1 + mod[m, 1]) * xh[0, r] + mod[m, 0], atol=1e-12)
    # scale = -1 makes every row equal to its mode's shift
    mod2 = mod.copy()
    mod2[:, 1] = -1.0
    np.testing.assert_allclose(o.modln(x, modes, mod2)[0], mod2[modes, 0], atol=1e-12)


def test_rms_norm_unit_rms():
    x = np.random.default_rng(5).normal(0, 3, size=(4, 24, 128))
    y = o.rms_norm(x, np.ones(128))
    np.testing.assert_allclose(np.sqrt((y * y).mean(-1)), 1.0, rtol=1e-6)
    w = np.random.default_rng(6).normal(size=128)
    np.testing.assert_allclose(o.rms_norm(x, w), y * w, atol=1e-12)


# ------------------------------------------------------------- RoPE

def test_rope_preserves_pair_norms():
    rng = np.random.default_rng(7)
    x = rng.normal(size=(9, 3, 128))
    pos = rng.integers(-20, 600, size=(9, 4)).astype(float)
    y = o.rope(x, pos)
    nx = x[..., 0::2] ** 2 + x[..., 1::2] ** 2
    ny = y[..., 0::2] ** 2 + y[..., 1::2] ** 2
    np.testing.assert_allclose(ny, nx, rtol=1e-12)


def test_rope_zero_position_is_identity():
    x = np.random.default_rng(8).normal(size=(5, 2, 128))
    np.testing.assert_array_equal(o.rope(x, np.zeros((5, 4))), x)


def test_rope_relative_property():
    rng = np.random.default_rng(9)
    q = rng.normal(size=(1, 1, 128))
    k = rng.normal(size=(1, 1, 128))
    p1 = np.array([[0.0, 3.0, 5.0, 7.0]])
    p2 = np.array([[0.0, 1.0, -2.0, 4.0]])
    d = p1 - p2
    a = np.sum(o.rope(q, p1) * o.rope(k, p2))
    b = np.sum(o.rope(q, d) * o.rope(k, np.zeros((1, 4))))
    assert a == pytest.approx(b, rel=1e-12)


def test_rope_axis_blocks_and_frequencies():
    # a position on one axis only rotates that axis' 32 dims; pair j of an
    # axis turns by p * 10000^(-2j/32)
    x = np.zeros((1, 1, 128))
    x[..., 0::2] = 1.0
    for axis in range(4):
        pos = np.zeros((1, 4))
        pos[0, axis] = 3.0
        y = o.rope(x, pos)[0, 0]
        for d in range(0, 128, 2):
            a, j = divmod(d // 2, 16)
            ang = 3.0 * 10000.0 ** (-2 * j / 32) if a == axis else 0.0
            assert y[d] == pytest.approx(math.cos(ang), abs=1e-14)
            assert y[d + 1] == pytest.approx(math.sin(ang), abs=1e-14)


# -------------------------------------------------------- attention

def test_attention_matches_library():
    rng = np.random.default_rng(10)
    q = rng.normal(size=(2, 13, 3, 128))
    k = rng.normal(size=(2, 17, 3, 128))
    v = rng.normal(size=(2, 17, 3, 128))
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q).transpose(1, 2), torch.from_numpy(k).transpose(1, 2),
        torch.from_numpy(v).transpose(1, 2)).transpose(1, 2).numpy()
    np.testing.assert_allclose(o.attention(q, k, v), ref, rtol=1e-10, atol=1e-12)


def test_attention_special_cases():
    rng = np.random.default_rng(11)
    k = rng.normal(size=(1, 6, 2, 128))
    v = rng.normal(size=(1, 6, 2, 128))
    # zero queries attend uniformly
    out = o.attention(np.zeros((1, 4, 2, 128)), k, v)
    np.testing.assert_allclose(out, np.broadcast_to(v.mean(1, keepdims=True), out.shape), atol=1e-14)
    # a single key returns its value
    out = o.attention(rng.normal(size=(1, 3, 2, 128)), k[:, :1], v[:, :1])
    np.testing.assert_allclose(out, np.broadcast_to(v[:, :1], out.shape), atol=1e-14)


def _brute_attention(q, k, v):
    # scalar loops on a tiny case
    Rq, Rk, d = q.shape[0], k.shape[0], q.shape[1]
    out = np.zeros((Rq, d))
    for i in range(Rq):
        s = [sum(q[i, c] * k[j, c] for c in range(d)) / math.sqrt(d) for j in range(Rk)]
        m = max(s)
        e = [math.exp(t - m) for t in s]
        z = sum(e)
        for j in range(Rk):
            out[i] += e[j] / z * v[j]
    return out


def test_attention_brute_force_tiny():
    rng = np.random.default_rng(12)
    q = rng.normal(size=(1, 4, 1, 128))
    k = rng.normal(size=(1, 5, 1, 128))
    v = rng.normal(size=(1, 5, 1, 128))
    np.testing.assert_allclose(o.attention(q, k, v)[0, :, 0], _brute_attention(q[0, :, 0], k[0, :, 0], v[0, :, 0]), atol=1e-12)


# ------------------------------------------------------------- block

@pytest.fixture(scope="module")
def small_block():
    w = ki.block_weights(0, "pin.block")
    n_txt, gh, gw = 6, 3, 4
    pos = o.positions(n_txt, (gh, gw))
    modes = o.mode_of_rows(n_txt, gh * gw, 0)
    x = ki.tokens(1, "pin", 1, len(modes)).astype(np.float64)
    mod = ki.modulation_vectors(1, "pin").astype(np.float64)
    return w, pos, modes, x, mod


def test_block_gate_zero_is_identity(small_block):
    w, pos, modes, x, mod = small_block
    m = mod.copy()
    m[:, 2] = 0.0
    np.testing.assert_array_equal(o.block(x, pos, modes, m, w), x)


def test_block_linear_in_gate(small_block):
    w, pos, modes, x, mod = small_block
    m2 = mod.copy()
    m2[:, 2] *= 2.0
    d1 = o.block(x, pos, modes, mod, w) - x
    d2 = o.block(x, pos, modes, m2, w) - x
    np.testing.assert_allclose(d2, 2 * d1, rtol=1e-9, atol=1e-9)


def test_block_constant_input_closed_form(small_block):
    # scale = -1: every row of h equals its mode's shift. Give all modes the
    # same shift c: all values are equal, so attention returns that value
    # whatever the scores, and the block delta is gate * (W_o (W_v c) + W_d swiglu).
    w, pos, modes, x, mod = small_block
    c = np.random.default_rng(13).normal(size=o.DIM)
    m = mod.copy()
    m[:, 1] = -1.0
    m[:, 0] = c
    D, F = o.DIM, o.MLP_HIDDEN
    w_in = w["w_in"].astype(np.float64)
    w_out = w["w_out"].astype(np.float64)
    v = w_in[2 * D:3 * D] @ c
    g = w_in[3 * D:3 * D + F] @ c
    u = w_in[3 * D + F:] @ c
    delta = w_out[:, :D] @ v + w_out[:, D:] @ (g / (1 + np.exp(-g)) * u)
    out = o.block(x, pos, modes, m, w)
    np.testing.assert_allclose(out - x, m[modes, 2][None] * delta[None, None], rtol=1e-9, atol=1e-9)


def test_block_zero_queries_attend_uniformly(small_block):
    # With the q projection zeroed, q = 0 after RMSNorm and RoPE; the
    # attention branch is then the mean value row through the out-projection.
    w, pos, modes, x, mod = small_block
    D = o.DIM
    wz = dict(w)
    wz["w_in"] = w["w_in"].copy()
    wz["w_in"][0:D] = 0.0
    wm = dict(wz)
    wm["w_out"] = w["w_out"].copy()
    wm["w_out"][:, D:] = 0.0          # attention branch only
    h = o.modln(x, modes, mod)
    vbar = (h[0] @ w["w_in"][2 * D:3 * D].astype(np.float64).T).mean(0)
    expect = mod[modes, 2] * (w["w_out"][:, :D].astype(np.float64) @ vbar)[None]
    np.testing.assert_allclose(o.block(x, pos, modes, mod, wm)[0] - x[0], expect, rtol=1e-9, atol=1e-9)


def test_block_permutation_equivariance(small_block):
    w, pos, modes, x, mod = small_block
    perm = np.random.default_rng(14).permutation(len(modes))
    a = o.block(x, pos, modes, mod, w)[:, perm]
    b = o.block(x[:, perm], pos[perm], modes[perm], mod, w)
    np.testing.assert_allclose(a, b, rtol=1e-10, atol=1e-10)


def test_block_row_subset(small_block):
    w, pos, modes, x, mod = small_block
    rows = np.array([0, 5, 7, 17])
    np.testing.assert_allclose(o.block(x, pos, modes, mod, w, rows=rows),
                               o.block(x, pos, modes, mod, w)[:, rows], rtol=1e-12, atol=1e-12)


# ------------------------------------------------------ sampler pieces

def test_euler_constant_velocity_lands_on_x0():
    rng = np.random.default_rng(15)
    x0 = rng.normal(size=(10, 128))
    eps = rng.normal(size=(10, 128))
    for steps in (1, 4, 16, 50):
        s = o.sigma_schedule(steps)
        x = eps.copy()
        for i in range(steps):
            x = o.euler_step(x, eps - x0, s[i], s[i + 1])
        np.testing.assert_allclose(x, x0, atol=1e-12)
        # x0 preview at sigma = 1 recovers x0 exactly from the true velocity
        np.testing.assert_allclose(o.x0_preview(eps, eps - x0, 1.0), x0, atol=1e-12)


def test_euler_zero_velocity():
    x = np.random.default_rng(16).normal(size=(3, 128))
    np.testing.assert_array_equal(o.euler_step(x, np.zeros_like(x), 0.7, 0.3), x)


def test_cfg_limits():
    rng = np.random.default_rng(17)
    vc, vu = rng.normal(size=(2, 5, 128))
    np.testing.assert_allclose(o.cfg_combine(vc, vu, 1.0), vc, rtol=0, atol=1e-14)
    np.testing.assert_array_equal(o.cfg_combine(vc, vu, 0.0), vu)
    np.testing.assert_allclose(o.cfg_combine(vc, vu, 3.5), vu + 3.5 * (vc - vu))


# ------------------------------------------------------------- stack

def test_stage1_streams_are_isolated():
    m = ki.ModelWeights(seed=0, distilled=False, n_stage1=1, n_joint=1)
    n_txt, gh, gw = 5, 2, 3
    pos = o.positions(n_txt, (gh, gw))
    text = ki.text_embeddings(1, 1, n_txt)
    lat_a = ki.noise_latents(2, gh * gw)
    lat_b = ki.noise_latents(3, gh * gw)
    sa, sb = {}, {}
    o.transformer(m, lat_a, text, None, pos, 0.8, None, stage1_out=sa)
    o.transformer(m, lat_b, text, None, pos, 0.3, None, stage1_out=sb)
    # text stage-1 output ignores the image's latents and noise level
    np.testing.assert_array_equal(sa["txt"], sb["txt"])
    assert not np.allclose(sa["img"], sb["img"])


# ------------------------------------------------ embedder, output layer

def test_time_embed_mlp_identity_layers():
    # With the first layer copying the 256 sinusoid values into the first 256
    # of 3072 units and the second layer the identity, the embedder's output
    # is SiLU of the sinusoid of 1000 sigma there and 0 elsewhere. At
    # sigma = 0 every cosine is 1 and every sine 0: SiLU(1) = 1/(1 + 1/e).
    w1 = np.zeros((o.DIM, o.TIME_FREQ_DIM))
    w1[:o.TIME_FREQ_DIM] = np.eye(o.TIME_FREQ_DIM)
    w2 = np.eye(o.DIM)
    e = o.time_embed_mlp(w1, w2, 0.0)
    np.testing.assert_allclose(e[:128], 1.0 / (1.0 + math.exp(-1.0)), rtol=0, atol=1e-15)
    np.testing.assert_array_equal(e[128:], 0.0)
    # sigma = 0.25 -> t = 250; unit 0 is cos(250 * 1), unit 128 is sin(250 * 1)
    e = o.time_embed_mlp(w1, w2, 0.25)
    for u, z in ((0, math.cos(250.0)), (128, math.sin(250.0)), (1, math.cos(250.0 * 10000 ** (-1 / 128)))):
        assert e[u] == pytest.approx(z / (1.0 + math.exp(-z)), abs=1e-12)
    np.testing.assert_array_equal(e[256:], 0.0)
    # the second layer acts after the activation: w2 = -I flips the sign
    np.testing.assert_allclose(o.time_embed_mlp(w1, -w2, 0.25), -e, rtol=0, atol=1e-15)


def test_output_layer_scale_minus_one_gives_the_shift():
    # final (shift, scale) with scale = -1: every image row of the modulated
    # LayerNorm equals the shift, so the velocity is W_final . shift on every
    # row whatever the rows were; a swapped (scale, shift) order or a dropped
    # modulation gives something else
    rng = np.random.default_rng(21)
    x = rng.normal(size=(2, 7, o.DIM)) * 3.0 + 1.0
    w = ki.linear(0, "pin.final_out", o.LATENT_CH, o.DIM).astype(np.float64)
    shift = rng.normal(size=o.DIM)
    fm = np.stack([shift, -np.ones(o.DIM)])
    v = o.output_layer(x, fm, w)
    np.testing.assert_allclose(v, np.broadcast_to(w @ shift, v.shape), rtol=1e-12, atol=1e-12)


def test_output_layer_normalises_rows():
    # shift = scale = 0: the velocity is LayerNorm(x) . W^T, and LayerNorm
    # removes any per-row affine change a + b x (b > 0; up to its eps of 1e-6
    # against the variance, b >= 1 keeps that below 5e-7 relative)
    rng = np.random.default_rng(22)
    z = rng.normal(size=(1, 5, o.DIM))
    w = ki.linear(0, "pin.final_out", o.LATENT_CH, o.DIM).astype(np.float64)
    fm = np.zeros((2, o.DIM))
    a = rng.normal(size=(1, 5, 1)) * 4.0
    b = 1.0 + np.exp(rng.normal(size=(1, 5, 1)))
    np.testing.assert_allclose(o.output_layer(a + b * z, fm, w), o.output_layer(z, fm, w), rtol=0, atol=2e-6)
    zn = (z - z.mean(-1, keepdims=True)) / z.std(-1, keepdims=True)
    np.testing.assert_allclose(o.output_layer(z, fm, w), zn @ w.T, rtol=1e-5, atol=1e-5)


# ------------------------------------------------- transformer assembly

_STACKS = {}


def _tiny_stack(n_stage1, n_joint, distilled=True, seed=0):
    """Seeded stacks of the model's width with few blocks; weights are
    generated once per session and shared (treat them as read-only)."""
    key = (n_stage1, n_joint, distilled, seed)
    if key not in _STACKS:
        _STACKS[key] = ki.ModelWeights(seed=seed, distilled=distilled, n_stage1=n_stage1, n_joint=n_joint)
    return _STACKS[key]


def test_transformer_without_blocks_is_the_output_layer_of_the_image_rows():
    # 0 + 0 blocks: nothing mixes tokens, so the velocity is the output layer
    # applied to the projected image latents alone; text and references
    # change nothing
    m = _tiny_stack(0, 0)
    n_txt, grid, refs = 6, (3, 4), ((2, 2),)
    pos = o.positions(n_txt, grid, refs)
    lat = ki.noise_latents(2, 12)
    rl = ki.ref_latents(1, 4)
    v = o.transformer(m, lat, ki.text_embeddings(1, 2, n_txt), rl, pos, 0.7, 0.4)
    fin = o.stage_modulations(m.misc, 0.7, 0.4)["final"]
    expect = o.output_layer(lat.astype(np.float64) @ m.misc["img_in"].astype(np.float64).T, fin, m.misc["final_out"])
    assert v.shape == (2, 12, o.LATENT_CH)
    np.testing.assert_allclose(v[0], expect, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(v[1], expect, rtol=1e-12, atol=1e-12)
    v2 = o.transformer(m, lat, ki.text_embeddings(5, 2, n_txt), None, o.positions(n_txt, grid), 0.7, 0.4)
    np.testing.assert_allclose(v2, v, rtol=1e-12, atol=1e-12)


def test_transformer_text_rows_are_a_set_with_their_positions():
    # permuting the text rows together with their positions permutes the
    # text stream (RoPE carries the order) and leaves the image velocity as
    # it was: stage 1 is equivariant, joint attention sums over keys, and
    # only image rows reach the output layer
    m = _tiny_stack(1, 1, distilled=False)
    n_txt, grid = 7, (2, 3)
    pos = o.positions(n_txt, grid)
    text = ki.text_embeddings(1, 1, n_txt)
    lat = ki.noise_latents(2, 6)
    perm = np.random.default_rng(23).permutation(n_txt)
    pos_p = pos.copy()
    pos_p[:n_txt] = pos[perm]
    a = o.transformer(m, lat, text, None, pos, 0.6, None)
    b = o.transformer(m, lat, text[:, perm], None, pos_p, 0.6, None)
    np.testing.assert_allclose(a, b, rtol=1e-9, atol=1e-9)
    # moving the text positions (not the rows) does change it
    pos_q = pos.copy()
    pos_q[:n_txt, 3] += 1.0 + np.arange(n_txt)
    assert not np.allclose(o.transformer(m, lat, text, None, pos_q, 0.6, None), a)


def test_transformer_references_are_context_rows_projected_by_ref_in():
    # Without stage 1 and with the reference modulation weights set to the
    # text ones, a reference row is a context row modulated at t = 0 like
    # text: giving the references as references equals appending their
    # projected latents (ref_in, not img_in) to the text with their
    # positions. A reference projected by img_in or modulated at the image
    # time would break the equality.
    base = _tiny_stack(0, 2)
    m = ki.ModelWeights(seed=0, distilled=True, n_stage1=0, n_joint=2)
    m._blocks = base._blocks
    m._misc = misc = dict(base.misc)
    for st in (1, 2):
        misc[f"mod{st}.ref"] = misc[f"mod{st}.txt"]
    n_txt, grid, refs = 5, (2, 3), ((2, 2), (1, 3))
    pos = o.positions(n_txt, grid, refs)
    text = ki.text_embeddings(1, 1, n_txt)
    lat = ki.noise_latents(2, 6)
    rl = ki.ref_latents(1, 7)
    a = o.transformer(m, lat, text, rl, pos, 0.8, 0.5)
    ref_rows = rl.astype(np.float64) @ misc["ref_in"].astype(np.float64).T
    text2 = np.concatenate([text.astype(np.float64), ref_rows[None]], axis=1)
    pos2 = np.concatenate([pos[:n_txt], pos[n_txt + 6:], pos[n_txt:n_txt + 6]])
    b = o.transformer(m, lat, text2, None, pos2, 0.8, 0.5)
    np.testing.assert_allclose(a, b, rtol=1e-9, atol=1e-9)
    # and the references do reach the image through the joint blocks only
    s1 = _tiny_stack(1, 0)
    c = o.transformer(s1, lat, text, rl, pos, 0.8, 0.5)
    d = o.transformer(s1, lat, text, ki.ref_latents(4, 7), pos, 0.8, 0.5)
    np.testing.assert_array_equal(c, d)
    assert not np.allclose(a, o.transformer(m, lat, text, ki.ref_latents(4, 7), pos, 0.8, 0.5))


# ----------------------------------------------------- the sampler loop

@pytest.mark.parametrize("distilled", [True, False])
def test_denoise_loop_with_exact_velocity_lands_on_x0(monkeypatch, distilled):
    # A stand-in denoiser that returns the straight-path velocity eps - x0
    # (for every batch item): the sampler must land on x0 exactly, for any
    # number of steps, after visiting the shifted schedule in order; the
    # distilled model is told sigma_next (0 on the last step), the base
    # model is not. With guidance the two items combine by v_u + g (v_c - v_u).
    rng = np.random.default_rng(24)
    x0 = rng.normal(size=(9, o.LATENT_CH))
    eps = rng.normal(size=(9, o.LATENT_CH))
    calls = []

    def stub(model, x, text, ref, pos, sigma, sigma_next, stage1_out=None):
        calls.append((float(sigma), sigma_next))
        np.testing.assert_allclose(x, x0 + sigma * (eps - x0), atol=1e-12)  # on the straight path
        v = eps - x0
        return np.stack([v, v + 7.0]) if text.shape[0] == 2 else v[None]

    import oracle.klein as ok
    monkeypatch.setattr(ok, "transformer", stub)
    m = ki.ModelWeights(seed=0, distilled=distilled, n_stage1=0, n_joint=0)
    m._misc = {"tt_mlp1": None} if distilled else {}   # the sampler only asks whether the target embedder exists
    for steps in (1, 4, 16):
        calls.clear()
        out = o.denoise(m, eps, np.zeros((1, 3, o.DIM)), None, None, steps)
        np.testing.assert_allclose(out, x0, atol=1e-12)
        sig = o.sigma_schedule(steps)
        assert [c[0] for c in calls] == pytest.approx(list(sig[:-1]), abs=0)
        nxt = [c[1] for c in calls]
        if distilled:
            assert nxt == pytest.approx(list(sig[1:]), abs=0) and nxt[-1] == 0.0
        else:
            assert all(n is None for n in nxt)
    # guidance 1 keeps the conditional velocity (the +7 offset is the uncond)
    out = o.denoise(m, eps, np.zeros((2, 3, o.DIM)), None, None, 4, cfg=1.0)
    np.testing.assert_allclose(out, x0, atol=1e-12)


def test_transformer_image_row_subset():
    # the velocity of a subset of image rows equals those rows of the full
    # velocity (the last joint block evaluates only the subset's outputs)
    m = _tiny_stack(1, 1, distilled=False)
    n_txt, grid = 7, (2, 3)
    pos = o.positions(n_txt, grid)
    text = ki.text_embeddings(1, 1, n_txt)
    lat = ki.noise_latents(2, 6)
    full = o.transformer(m, lat, text, None, pos, 0.6, None)
    rows = np.array([0, 3, 5])
    sub = o.transformer(m, lat, text, None, pos, 0.6, None, img_rows=rows)
    np.testing.assert_allclose(sub, full[:, rows], rtol=1e-12, atol=1e-12)
    m0 = _tiny_stack(0, 0)
    np.testing.assert_allclose(o.transformer(m0, lat, text, None, pos, 0.6, 0.2, img_rows=rows),
                               o.transformer(m0, lat, text, None, pos, 0.6, 0.2)[:, rows], rtol=1e-12, atol=1e-12)
