"""Float64 CPU restatement of the FLUX.3 Image Klein denoiser.

TEST INFRASTRUCTURE ONLY (see the package docstring): imported by tests/,
the smoke check and the benchmark's CPU baseline, never by the product path.

Sources, cited by page and section:
  [blog]   "FLUX.3 Image Klein Is Now Available in Diffusers" (Diffusers
           release blog, English retelling), section "Speed, architecture,
           and how the tokens move".
  [blogzh] the Chinese translation of the same blog, with its block
           pseudo-code (``def block(x, shift, scale, gate)``) and its RoPE
           position table (text / image / reference rows).
  [guide]  "How to Run FLUX 3 Image Klein Locally", sections "The latent
           space and the VAE", "Inside the transformer", "The denoise loop",
           "What step distillation removed", "Why dropping CFG halves the
           compute", "The text encoder".
  [zh5]    the Chinese summary page (reference tokens offset negatively along l).

Readings taken where the pages are silent are marked READING and listed in
the design notes: LayerNorm/RMSNorm eps 1e-6; sinusoid [cos, sin] with
frequencies 10000^(-j/128); embedder Linear-SiLU-Linear; modulation
W * SiLU(e); chunk order (shift, scale, gate); RoPE rotates adjacent pairs
(2j, 2j+1) of each 32-dim axis block with angle p * theta^(-2j/32), axes in
the order (t, h, w, l); image position = integer token-grid index; SwiGLU
gate is the first half of the MLP-in output; attention has an output
projection; all references form one stage-1 stream.

Everything is float64. Inputs (weights, activations) are float32 arrays of
bf16-representable values from ``klein_inputs`` and are upcast on entry.
"""
from __future__ import annotations

import math

import numpy as np

from .fp8 import dequantize as fp8_dequantize
from .fp8 import fake_quant as fp8_fake_quant
from .nvfp4 import dequantize as nvfp4_dequantize
from .nvfp4 import fake_quant_rows as nvfp4_fake_quant_rows

DIM = 3072
HEADS = 24
HEAD_DIM = 128
MLP_HIDDEN = 9216
LATENT_CH = 128
TIME_FREQ_DIM = 256
AXES = 4
AXIS_DIM = 32
ROPE_THETA = 10000.0
SHIFT = 6.93
N_STAGE1 = 5
N_JOINT = 28
TEXT_PAD = 80
PATCH_PX = 16
LN_EPS = 1e-6
RMS_EPS = 1e-6
MODE_TXT, MODE_IMG, MODE_REF = 0, 1, 2
F64 = np.float64


# ---------------------------------------------------------------------------
# Sequence geometry
# ---------------------------------------------------------------------------

def image_tokens(height_px: int, width_px: int) -> int:
    """Tokens of a height x width image.

    [blog] / [guide] "The latent space and the VAE": the VAE downsamples 8x
    per side to 32 channels, then each 2x2 latent patch is one 128-channel
    token, so one token covers 16x16 pixels.
    """
    return (height_px // PATCH_PX) * (width_px // PATCH_PX)


def pad_text_len(n: int) -> int:
    """[blog] / [guide] "The text encoder": prompts are padded to a multiple of 80."""
    return int(math.ceil(n / TEXT_PAD) * TEXT_PAD) if n > 0 else 0


def positions(n_txt: int, img_hw: tuple, refs: tuple = ()) -> np.ndarray:
    """(t, h, w, l) position per token of the [text | image | refs...] sequence.

    [blogzh] RoPE table: text token i -> (0, 0, 0, i); image token at
    (row, col) -> (0, row/2, col/2, 0); reference k at (row, col) ->
    (0, row/2, col/2, -(k+1)). READING: row/2, col/2 of the latent-pixel grid
    is the integer index on the token grid, rows scanned row-major.
    """
    rows = []
    for i in range(n_txt):
        rows.append((0.0, 0.0, 0.0, float(i)))
    gh, gw = img_hw
    for r in range(gh):
        for c in range(gw):
            rows.append((0.0, float(r), float(c), 0.0))
    for k, (rh, rw) in enumerate(refs):
        for r in range(rh):
            for c in range(rw):
                rows.append((0.0, float(r), float(c), float(-(k + 1))))
    return np.array(rows, dtype=F64).reshape(-1, AXES)


# ---------------------------------------------------------------------------
# Schedule, Euler, guidance
# ---------------------------------------------------------------------------

def sigma_schedule(steps: int, shift: float = SHIFT) -> np.ndarray:
    """Shifted noise levels sigma_0..sigma_steps (last = 0).

    [guide] "The denoise loop": start from `steps` levels evenly spaced from
    1 down to 1/steps, shift each with s*sigma / (1 + (s-1)*sigma), and jump
    to 0 after the last one.
    """
    base = np.linspace(1.0, 1.0 / steps, steps, dtype=F64)
    shifted = shift * base / (1.0 + (shift - 1.0) * base)
    return np.concatenate([shifted, [0.0]])


def timesteps(sigmas: np.ndarray) -> np.ndarray:
    """[blogzh] preview step: timesteps are sigmas scaled to [0, 1000]."""
    return 1000.0 * np.asarray(sigmas, dtype=F64)


def euler_step(x: np.ndarray, v: np.ndarray, sigma: float, sigma_next: float) -> np.ndarray:
    """[guide] "The denoise loop": the latent moves by (sigma_next - sigma) * v."""
    return np.asarray(x, F64) + (sigma_next - sigma) * np.asarray(v, F64)


def x0_preview(x: np.ndarray, v: np.ndarray, sigma: float) -> np.ndarray:
    """[guide] "The denoise loop" / [blogzh] preview block: x0 = x - sigma * v."""
    return np.asarray(x, F64) - sigma * np.asarray(v, F64)


def cfg_combine(v_cond: np.ndarray, v_uncond: np.ndarray, g: float) -> np.ndarray:
    """[guide] "Why dropping CFG halves the compute": v = v_u + g (v_c - v_u)."""
    v_c = np.asarray(v_cond, F64)
    v_u = np.asarray(v_uncond, F64)
    return v_u + g * (v_c - v_u)


# ---------------------------------------------------------------------------
# Timestep embedding and modulation
# ---------------------------------------------------------------------------

def silu(x):
    x = np.asarray(x, F64)
    return x / (1.0 + np.exp(-x))


def timestep_sinusoid(t: float) -> np.ndarray:
    """256-dim sinusoidal embedding of a scalar timestep t (already x1000).

    READING: [cos(t f_j) for j<128] + [sin(t f_j) for j<128], f_j = 10000^(-j/128).
    """
    half = TIME_FREQ_DIM // 2
    f = np.power(10000.0, -np.arange(half, dtype=F64) / half)
    a = float(t) * f
    return np.concatenate([np.cos(a), np.sin(a)])


def time_embed_mlp(w1: np.ndarray, w2: np.ndarray, sigma: float) -> np.ndarray:
    """Two-layer bias-free embedder of sigma (guide, "What step distillation
    removed": 256 x 3072 + 3072 x 3072 weights, no biases). READING: SiLU between."""
    s = timestep_sinusoid(1000.0 * sigma)
    return np.asarray(w2, F64) @ silu(np.asarray(w1, F64) @ s)


def time_embedding(misc: dict, sigma: float, sigma_next: float | None) -> np.ndarray:
    """Embedding e for a token stream at noise level sigma.

    [guide] "What step distillation removed": the distilled model embeds the
    target level with a second embedder and adds it to every mode's
    modulation input.
    """
    e = time_embed_mlp(misc["t_mlp1"], misc["t_mlp2"], sigma)
    if "tt_mlp1" in misc and sigma_next is not None:
        e = e + time_embed_mlp(misc["tt_mlp1"], misc["tt_mlp2"], sigma_next)
    return e


def modulation(w_mod: np.ndarray, e: np.ndarray, n_chunks: int) -> np.ndarray:
    """READING: W * SiLU(e), split into n_chunks vectors of DIM in the order
    shift, scale, gate (the argument order of the [blogzh] block pseudo-code)."""
    out = np.asarray(w_mod, F64) @ silu(e)
    return out.reshape(n_chunks, DIM)


def stage_modulations(misc: dict, sigma: float, sigma_next: float | None) -> dict:
    """Per-stage, per-mode (shift, scale, gate), plus the final (shift, scale).

    [blog]: image tokens use the current t; text and reference tokens always
    use t = 0. Each mode has its own scale, shift and gate.
    """
    e_img = time_embedding(misc, sigma, sigma_next)
    e_ctx = time_embedding(misc, 0.0, sigma_next)
    out = {}
    for stage in (1, 2):
        out[stage] = np.stack([
            modulation(misc[f"mod{stage}.txt"], e_ctx, 3),
            modulation(misc[f"mod{stage}.img"], e_img, 3),
            modulation(misc[f"mod{stage}.ref"], e_ctx, 3),
        ])
    out["final"] = modulation(misc["final_mod"], e_img, 2)
    return out


# ---------------------------------------------------------------------------
# Block pieces
# ---------------------------------------------------------------------------

def layer_norm(x: np.ndarray) -> np.ndarray:
    """LayerNorm over the last axis with no learned scale or shift ([blog])."""
    x = np.asarray(x, F64)
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + LN_EPS)


def modulate(xhat: np.ndarray, shift: np.ndarray, scale: np.ndarray) -> np.ndarray:
    """[blogzh] block pseudo-code: the normalised row times (1 + scale), plus shift."""
    return (1.0 + scale) * xhat + shift


def modln(x: np.ndarray, mode_of_row: np.ndarray, mod: np.ndarray) -> np.ndarray:
    """Modulated LayerNorm of x [..., R, DIM] with per-row mode.

    mod: [3 modes, >=2, DIM] with chunk 0 = shift, 1 = scale.
    """
    shift = mod[mode_of_row, 0]
    scale = mod[mode_of_row, 1]
    return modulate(layer_norm(x), shift, scale)


def rms_norm(x: np.ndarray, w: np.ndarray) -> np.ndarray:
    """RMS-normalise the last axis (one head, 128 dims) and scale by w ([blog])."""
    x = np.asarray(x, F64)
    return x / np.sqrt((x * x).mean(axis=-1, keepdims=True) + RMS_EPS) * np.asarray(w, F64)


def rope_angles(pos: np.ndarray, theta: float = ROPE_THETA) -> np.ndarray:
    """Rotation angle per (token, pair): [R, 64].

    [blog] RoPE paragraph: four axes (t, h, w, l), 32 of the 128 head dims
    each. Pair p = 16*axis + j covers dims (2p, 2p+1); READING: its angle is
    pos[axis] * theta^(-2j/32).
    """
    pos = np.asarray(pos, F64)
    j = np.arange(AXIS_DIM // 2, dtype=F64)
    freq = np.power(theta, -2.0 * j / AXIS_DIM)
    ang = pos[:, :, None] * freq[None, None, :]
    return ang.reshape(pos.shape[0], AXES * AXIS_DIM // 2)


def rope(x: np.ndarray, pos: np.ndarray, theta: float = ROPE_THETA) -> np.ndarray:
    """Rotate x [..., R, heads, 128] by the positions pos [R, 4]."""
    x = np.asarray(x, F64)
    ang = rope_angles(pos, theta)[:, None, :]
    c, s = np.cos(ang), np.sin(ang)
    x0 = x[..., 0::2]
    x1 = x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = x0 * c - x1 * s
    out[..., 1::2] = x0 * s + x1 * c
    return out


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray) -> np.ndarray:
    """Full softmax attention, no mask, scale 1/sqrt(128).

    q: [B, Rq, heads, 128]; k, v: [B, Rk, heads, 128] -> [B, Rq, heads, 128].
    [blog]: in stage 2 every token attends to every token; the padding of
    the text is attended too.
    """
    q = np.asarray(q, F64)
    k = np.asarray(k, F64)
    v = np.asarray(v, F64)
    B, Rq, H, Dh = q.shape
    out = np.empty((B, Rq, H, Dh), dtype=F64)
    scale = 1.0 / math.sqrt(Dh)
    for b in range(B):
        for h in range(H):
            s = (q[b, :, h, :] @ k[b, :, h, :].T) * scale
            s = s - s.max(axis=1, keepdims=True)
            p = np.exp(s)
            p = p / p.sum(axis=1, keepdims=True)
            out[b, :, h, :] = p @ v[b, :, h, :]
    return out


def swiglu(g: np.ndarray, u: np.ndarray) -> np.ndarray:
    """READING: SwiGLU hidden = silu(gate half) * (up half)."""
    return silu(g) * np.asarray(u, F64)


def _split_w_in(w_in):
    w = np.asarray(w_in, F64)
    return (w[0:DIM], w[DIM:2 * DIM], w[2 * DIM:3 * DIM],
            w[3 * DIM:3 * DIM + MLP_HIDDEN], w[3 * DIM + MLP_HIDDEN:])


def block(x: np.ndarray, pos: np.ndarray, mode_of_row: np.ndarray, mod: np.ndarray,
          w: dict, rows: np.ndarray | None = None) -> np.ndarray:
    """One block ([blogzh] block pseudo-code; [guide] "Inside the transformer").

    x [B, R, DIM]; pos [R, 4]; mode_of_row [R] in {0 txt, 1 img, 2 ref};
    mod [3, 3, DIM] per-mode (shift, scale, gate); w from klein_inputs.
    Steps: the no-affine LayerNorm of x is modulated by the row's mode
    (times 1 + scale, plus shift); that one normalised input feeds both the
    query/key/value projections and the SwiGLU MLP; q and k are RMS-normed
    per head and rotated by RoPE; the attention output (through its output
    projection) and the MLP output are summed, multiplied by the row's gate
    and added to x.
    If `rows` is given, only those output rows are computed (all rows still
    supply keys and values); the result is [B, len(rows), DIM].

    Rowwise FP8 weights (keys w_in_q/w_in_s/w_out_q/w_out_s, from
    oracle.fp8.quantize_block_weights): the weights are dequantised, and the
    two GEMM inputs, the normalised rows h and the concatenated
    [attention heads | SwiGLU hidden] rows, are quantised rowwise to e4m3
    and dequantised before their GEMM (oracle.fp8 states the reading).
    NVFP4 weights (keys w_in_nv/w_out_nv, from
    oracle.nvfp4.quantize_block_weights): the same two inputs go through NVFP4
    with one second-level scale per row (oracle.nvfp4 states the reading).
    """
    x = np.asarray(x, F64)
    B, R, _ = x.shape
    if rows is None:
        rows = np.arange(R)
    rows = np.asarray(rows)
    fp8 = "w_in_q" in w
    nv = "w_in_nv" in w
    h = modln(x, mode_of_row, mod)
    if fp8:
        h = fp8_fake_quant(h)
        w_in = fp8_dequantize(w["w_in_q"], w["w_in_s"])
        w_out = fp8_dequantize(w["w_out_q"], w["w_out_s"])
    elif nv:
        h = nvfp4_fake_quant_rows(h)
        w_in = nvfp4_dequantize(*w["w_in_nv"])
        w_out = nvfp4_dequantize(*w["w_out_nv"])
    else:
        w_in = w["w_in"]
        w_out = np.asarray(w["w_out"], F64)
    w_q, w_k, w_v, w_g, w_u = _split_w_in(w_in)
    hr = h[:, rows]
    q = (hr @ w_q.T).reshape(B, len(rows), HEADS, HEAD_DIM)
    k = (h @ w_k.T).reshape(B, R, HEADS, HEAD_DIM)
    v = (h @ w_v.T).reshape(B, R, HEADS, HEAD_DIM)
    q = rope(rms_norm(q, w["q_norm"]), pos[rows])
    k = rope(rms_norm(k, w["k_norm"]), pos)
    heads = attention(q, k, v).reshape(B, len(rows), DIM)
    hidden = swiglu(hr @ w_g.T, hr @ w_u.T)
    if fp8 or nv:
        # READING (quantised files): the two down-projections take one
        # rowwise-quantised input, the [attention heads | SwiGLU hidden] row,
        # with a single scale across both parts.
        a_cat = np.concatenate([heads, hidden], axis=-1)
        a_cat = fp8_fake_quant(a_cat) if fp8 else nvfp4_fake_quant_rows(a_cat)
        out = a_cat @ w_out.T
    else:
        # [blogzh] block pseudo-code: attention output (through its output
        # projection) plus the MLP output
        w_o = np.asarray(w_out[:, :DIM], F64)
        w_d = np.asarray(w_out[:, DIM:], F64)
        out = heads @ w_o.T + hidden @ w_d.T
    gate = mod[mode_of_row[rows], 2]
    return x[:, rows] + gate * out


def output_layer(x_img: np.ndarray, final_mod: np.ndarray, w_final: np.ndarray) -> np.ndarray:
    """Image tokens only: modulated no-affine LayerNorm (final shift, scale),
    then Linear 3072 -> 128 ([guide] "Inside the transformer"; READING on the
    final modulation, from the parameter count)."""
    h = modulate(layer_norm(x_img), final_mod[0], final_mod[1])
    return h @ np.asarray(w_final, F64).T


# ---------------------------------------------------------------------------
# The transformer and the sampler
# ---------------------------------------------------------------------------

def mode_of_rows(n_txt: int, n_img: int, n_ref: int) -> np.ndarray:
    return np.concatenate([np.full(n_txt, MODE_TXT), np.full(n_img, MODE_IMG),
                           np.full(n_ref, MODE_REF)]).astype(np.int64)


def transformer(model, latents: np.ndarray, text: np.ndarray, ref_lat: np.ndarray | None,
                pos: np.ndarray, sigma: float, sigma_next: float | None,
                stage1_out: dict | None = None, img_rows: np.ndarray | None = None) -> np.ndarray:
    """One denoiser call: velocity for the image tokens, [B, n_img, 128].

    [blog] two stages: stage 1 runs each stream (text, image, references)
    through its own 5 blocks attending only to itself; stage 2 concatenates
    [text | image | reference] and runs 28 shared blocks over everything;
    then text and reference tokens are dropped and the image tokens go
    through the output layer.

    model: klein_inputs.ModelWeights. latents [n_img, 128] (shared by the
    batch), text [B, n_txt, DIM] or, when the model has the text input
    projection, the stacked encoder hidden states [B, n_txt, 8 * 2560]
    ([blog] / [guide] "The text encoder": hidden states of eight encoder
    layers are stacked per token and projected linearly to the model width),
    ref_lat [n_ref, 128] or None.
    If stage1_out is a dict, the stage-1 outputs per stream are stored in it.
    If img_rows (indices into the image tokens) is given, only those rows of
    the velocity are computed, [B, len(img_rows), 128]: the last joint block
    evaluates just those output rows (every row still supplies keys and
    values), as block() does for a row subset.
    """
    misc = model.misc
    text = np.asarray(text, F64)
    if "txt_in" in misc:
        text = text @ np.asarray(misc["txt_in"], F64).T
    B, n_txt, _ = text.shape
    n_img = latents.shape[0]
    n_ref = 0 if ref_lat is None else ref_lat.shape[0]
    mods = stage_modulations(misc, sigma, sigma_next)

    img = np.asarray(latents, F64) @ np.asarray(misc["img_in"], F64).T
    streams = {"txt": text,
               "img": np.broadcast_to(img, (B, n_img, DIM)).copy()}
    bounds = {"txt": (0, n_txt), "img": (n_txt, n_txt + n_img),
              "ref": (n_txt + n_img, n_txt + n_img + n_ref)}
    if n_ref:
        ref = np.asarray(ref_lat, F64) @ np.asarray(misc["ref_in"], F64).T
        streams["ref"] = np.broadcast_to(ref, (B, n_ref, DIM)).copy()
    modes = mode_of_rows(n_txt, n_img, n_ref)

    for name, s in list(streams.items()):
        lo, hi = bounds[name]
        for w in model.stage1(name):
            s = block(s, pos[lo:hi], modes[lo:hi], mods[1], w)
        streams[name] = s
    if stage1_out is not None:
        stage1_out.update(streams)

    x = np.concatenate([streams[k] for k in ("txt", "img", "ref") if k in streams], axis=1)
    joint = model.joint()
    if img_rows is None:
        for w in joint:
            x = block(x, pos, modes, mods[2], w)
        return output_layer(x[:, n_txt:n_txt + n_img], mods["final"], misc["final_out"])
    out_rows = n_txt + np.asarray(img_rows)
    for i, w in enumerate(joint):
        last = i == len(joint) - 1
        x = block(x, pos, modes, mods[2], w, rows=out_rows if last else None)
    if not joint:
        x = x[:, out_rows]
    return output_layer(x, mods["final"], misc["final_out"])


def denoise(model, noise: np.ndarray, text: np.ndarray, ref_lat: np.ndarray | None,
            pos: np.ndarray, steps: int, cfg: float = 1.0, shift: float = SHIFT,
            on_step=None) -> np.ndarray:
    """Flow-matching Euler sampler ([guide] "The denoise loop").

    Starts at sigma = 1 from `noise` [n_img, 128]. With cfg > 1, `text` holds
    [cond, uncond] and each step runs both and combines them ([guide] "Why
    dropping CFG halves the compute"). The distilled model (misc has the
    target embedder) is told sigma_next each step.
    """
    sig = sigma_schedule(steps, shift)
    x = np.asarray(noise, F64).copy()
    distilled = "tt_mlp1" in model.misc
    for i in range(steps):
        s_next = sig[i + 1] if distilled else None
        v = transformer(model, x, text, ref_lat, pos, sig[i], s_next)
        if cfg > 1.0:
            v = cfg_combine(v[0], v[1], cfg)
        else:
            v = v[0]
        x_new = euler_step(x, v, sig[i], sig[i + 1])
        if on_step is not None:
            on_step(i, x, v, sig[i])
        x = x_new
    return x


# ---------------------------------------------------------------------------
# Structure
# ---------------------------------------------------------------------------

def parameter_count(distilled: bool, n_stage1: int = N_STAGE1, n_joint: int = N_JOINT,
                    txt_in: bool = True) -> int:
    """Parameters of the transformer as this oracle lays it out.

    Blocks: fused in-projection (q, k, v, gate, up), fused out-projection
    (attention out + MLP down), q/k norm weights; per-mode stage-1 blocks for
    3 streams plus the joint blocks; text (20480 -> 3072), image and reference
    input projections; final Linear 3072 -> 128; timestep embedder; per-mode,
    per-stage modulation and final modulation; optional target embedder.
    [guide] "What step distillation removed" prints the totals.
    """
    blk = DIM * (3 * DIM + 2 * MLP_HIDDEN) + (DIM + MLP_HIDDEN) * DIM + 2 * HEAD_DIM
    n = (3 * n_stage1 + n_joint) * blk
    n += (8 * 2560 * DIM if txt_in else 0) + 2 * LATENT_CH * DIM + DIM * LATENT_CH
    n += TIME_FREQ_DIM * DIM + DIM * DIM
    n += 2 * 3 * 3 * DIM * DIM + 2 * DIM * DIM
    if distilled:
        n += TIME_FREQ_DIM * DIM + DIM * DIM
    return n
