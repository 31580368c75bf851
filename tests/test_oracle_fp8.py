"""Pins for the oracle's rowwise FP8 (e4m3) quantisation.

The e4m3 format is fixed by the OCP 8-bit floating point definition; the
encoder and decoder are checked against torch's float8_e4m3fn conversion (an
independent library routine) over every code, random values across the whole
range, and every tie; the rowwise quantiser against the properties its
definition fixes (the row maximum lands on 448, the error bound of a 3-bit
mantissa, exact round trips, the scale axis); the FP8 block against the exact
block within the error that quantisation allows.
"""
import numpy as np
import pytest

import klein_inputs as ki
import oracle as o
from oracle import fp8

torch = pytest.importorskip("torch")


def _torch_decode(codes):
    return torch.from_numpy(np.asarray(codes, np.uint8)).view(torch.float8_e4m3fn).double().numpy()


def _torch_encode(x32):
    return torch.from_numpy(np.asarray(x32, np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_decode_every_code_matches_library():
    c = np.arange(256, dtype=np.uint8)
    got, ref = fp8.e4m3_decode(c), _torch_decode(c)
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    assert np.isnan(got).sum() == 2           # S.1111.111 only
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok])


def test_encode_random_values_match_library():
    rng = np.random.default_rng(7)
    x = (rng.standard_normal(100000) * np.exp(rng.uniform(-16, 6.2, 100000))).astype(np.float32)
    x = x[np.abs(x) <= 448]
    assert np.array_equal(fp8.e4m3_encode(x), _torch_encode(x))


def test_encode_ties_round_to_even():
    vals = fp8.e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8))       # 0 .. 448, ascending
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)
    assert np.all(mids.astype(np.float64) == (vals[:-1] + vals[1:]) / 2)   # exact in fp32
    got = fp8.e4m3_encode(mids)
    assert np.array_equal(got, _torch_encode(mids))
    assert np.all(got % 2 == 0)               # every tie lands on the even code
    got_neg = fp8.e4m3_encode(-mids)
    assert np.array_equal(got_neg, got | 0x80)


def test_encode_worked_values():
    x = np.array([1.0, -1.0, 448.0, 1000.0, 464.0, 2.0 ** -9, 2.0 ** -10, 3 * 2.0 ** -10,
                  2.0 ** -6, 0.0, -0.0, np.inf, -np.inf, np.nan], np.float32)
    want = [0x38, 0xB8, 0x7E, 0x7E, 0x7E, 0x01, 0x00, 0x02, 0x08, 0x00, 0x80, 0x7E, 0xFE, 0x7F]
    assert fp8.e4m3_encode(x).tolist() == want


def test_rowwise_max_lands_on_448_and_error_bound():
    rng = np.random.default_rng(3)
    mag = np.exp(rng.uniform(-8, 8, (64, 1)))
    x = (rng.standard_normal((64, 3072)) * mag).astype(np.float32)
    codes, scale = fp8.quantize_rowwise(x)
    assert codes.dtype == np.uint8 and scale.dtype == np.float32 and scale.shape == (64,)
    dec = fp8.e4m3_decode(codes)
    assert np.all(np.max(np.abs(dec), axis=1) == 448.0)
    # the scale follows each row's own magnitude (rowwise, not columnwise)
    amax = np.max(np.abs(x), axis=1)
    assert np.allclose(scale, amax / 448.0, rtol=1e-7)
    err = np.abs(fp8.dequantize(codes, scale) - x)
    # half a unit of the 3-bit mantissa, or half the subnormal step, plus float32 rounding
    bound = np.maximum(2.0 ** -4 * np.abs(x), 2.0 ** -10 * scale[:, None]) * (1 + 1e-6) + 1e-6 * np.abs(x)
    assert np.all(err <= bound)


def test_rowwise_exact_round_trip_and_zero_row():
    rng = np.random.default_rng(4)
    codes = rng.integers(0, 0x7E, (8, 256)).astype(np.uint8) | (rng.integers(0, 2, (8, 256)) * 0x80).astype(np.uint8)
    codes[:, 0] = 0x7E                        # each row reaches 448
    p2 = 2.0 ** rng.integers(-20, 20, 8)
    x = (fp8.e4m3_decode(codes) * p2[:, None]).astype(np.float32)
    x = np.vstack([x, np.zeros((1, 256), np.float32)])
    q, s = fp8.quantize_rowwise(x)
    assert np.array_equal(fp8.dequantize(q, s), x.astype(np.float64))
    assert s[-1] == 0 and not q[-1].any()


def test_weight_quantisation_is_per_output_channel():
    w = ki.block_weights(0, "fp8pin")
    wq = fp8.quantize_block_weights(w)
    assert wq["w_in_q"].shape == (3 * ki.DIM + 2 * ki.MLP_HIDDEN, ki.DIM)
    assert wq["w_in_s"].shape == (3 * ki.DIM + 2 * ki.MLP_HIDDEN,)
    assert wq["w_out_q"].shape == (ki.DIM, ki.DIM + ki.MLP_HIDDEN)
    assert wq["w_out_s"].shape == (ki.DIM,)
    # w_out's two halves have different fan-in, so its row amax comes from the
    # larger-spread half; every row scale matches its own row
    assert np.allclose(wq["w_out_s"], np.max(np.abs(w["w_out"]), axis=1) / 448.0, rtol=1e-7)


def test_fp8_block_tracks_exact_block():
    w = ki.block_weights(0, "joint.0")
    wq = fp8.quantize_block_weights(w)
    x = ki.tokens(1, "fp8blk", 1, 144)
    pos = o.positions(80, (8, 8))
    modes = o.mode_of_rows(80, 64, 0)
    mod = ki.modulation_vectors(1, "fp8blk")
    exact = o.block(x, pos, modes, mod, w)
    quant = o.block(x, pos, modes, mod, wq)
    d_e, d_q = exact - x, quant - x
    rel = np.sqrt(np.mean((d_q - d_e) ** 2) / np.mean(d_e ** 2))
    # each e4m3 operand carries at most 2^-4 relative error, about 0.026 RMS
    # for a rounding error uniform over the 3-bit mantissa step; four quantised
    # operands (h, W_in, the concatenated rows, W_out) whose errors add
    # incoherently give ~0.05 RMS on the block's update before RMSNorm, softmax
    # and SwiGLU reshape it (0.064 here); a wrong scale axis or a dropped scale
    # gives O(1).
    assert 0.02 < rel < 0.1, rel
    cos = np.sum(d_q * d_e) / np.sqrt(np.sum(d_q ** 2) * np.sum(d_e ** 2))
    assert cos > 0.997, cos


def test_quantized_model_transformer_tracks_exact():
    m = ki.ModelWeights(seed=0, distilled=True, n_stage1=1, n_joint=1)
    qm = fp8.QuantizedModel(m)
    lat = ki.noise_latents(2, 16)
    text = ki.text_embeddings(1, 1, 20)
    pos = o.positions(20, (4, 4))
    v_e = o.transformer(m, lat, text, None, pos, 0.7, 0.5)
    v_q = o.transformer(qm, lat, text, None, pos, 0.7, 0.5)
    cos = np.sum(v_e * v_q) / np.sqrt(np.sum(v_e ** 2) * np.sum(v_q ** 2))
    assert cos > 0.99, cos
    assert not np.array_equal(v_e, v_q)


# The GPU's FP8 block keeps the [attention | SwiGLU] rows in bf16 before it
# quantises them; this measures, on the oracle alone, what one bf16 rounding
# at that point does to the block (the GPU parity test's bound is derived from
# it): the update's relative RMS error and the worst element against RMS(output).
FP8_STORAGE_REL_MAX = 0.03
FP8_STORAGE_WORST_MAX = 0.09   # 0.083 measured; the GPU test allows 0.12


def test_fp8_block_sensitivity_to_bf16_storage_of_the_out_projection_input():
    from oracle.klein import DIM, HEAD_DIM, HEADS, _split_w_in, attention, modln, rms_norm, rope, swiglu
    w = ki.block_weights(0, "joint.0")
    wq = fp8.quantize_block_weights(w)
    x = ki.tokens(1, "fp8block.config1", 1, 144)
    mod = ki.modulation_vectors(1, "fp8block.config1").astype(np.float64)
    pos = o.positions(80, (8, 8))
    modes = o.mode_of_rows(80, 64, 0)
    ref = o.block(x, pos, modes, mod, wq)
    # the same block, recomposed from the oracle's steps, with the
    # concatenated rows rounded to bf16 before their quantisation
    h = fp8.fake_quant(modln(x, modes, mod))
    w_q, w_k, w_v, w_g, w_u = _split_w_in(fp8.dequantize(wq["w_in_q"], wq["w_in_s"]))
    q = rope(rms_norm((h @ w_q.T).reshape(1, 144, HEADS, HEAD_DIM), w["q_norm"]), pos)
    k = rope(rms_norm((h @ w_k.T).reshape(1, 144, HEADS, HEAD_DIM), w["k_norm"]), pos)
    v = (h @ w_v.T).reshape(1, 144, HEADS, HEAD_DIM)
    a_cat = np.concatenate([attention(q, k, v).reshape(1, 144, DIM), swiglu(h @ w_g.T, h @ w_u.T)], -1)
    same = x + mod[modes, 2] * (fp8.fake_quant(a_cat) @ fp8.dequantize(wq["w_out_q"], wq["w_out_s"]).T)
    assert np.max(np.abs(same - ref)) <= 1e-9 * np.sqrt(np.mean(ref ** 2))   # the recomposition is the block
    a_bf = ki.round_to_bf16(a_cat.astype(np.float32)).astype(np.float64)
    pert = x + mod[modes, 2] * (fp8.fake_quant(a_bf) @ fp8.dequantize(wq["w_out_q"], wq["w_out_s"]).T)
    r = lambda a: float(np.sqrt(np.mean(a * a)))
    rel = r(pert - ref) / r(ref - x)
    worst = float(np.max(np.abs(pert - ref))) / r(ref)
    assert 0.003 < rel <= FP8_STORAGE_REL_MAX, rel
    assert 0.01 < worst <= FP8_STORAGE_WORST_MAX, worst
