"""Seeded synthetic inputs shared by the CPU oracle and the GPU harness.

This module only draws numbers. It holds none of the denoiser's arithmetic:
every tensor is an independent draw from numpy's PCG64 generator, keyed by a
base seed and the tensor's name, so that any one tensor can be produced
without producing the others. Values are rounded to the nearest bfloat16
(ties to even) and returned as float32, so the GPU path (which stores these
tensors as bf16) and the oracle (which upcasts them) read the very same
numbers.

Recipe (FLUX.3 Image Klein model shapes; random init stands in for trained
weights, which are not available):
  * Linear weights ~ N(0, std = 1/sqrt(fan_in)), stored [out, in].
  * QK-RMSNorm weights ~ 1 + 0.1 * N(0, 1).
  * Activations, text embeddings, noise and reference latents ~ N(0, 1).
  * Weights use seed 0, activations seed 1, noise seed 2 by default.
"""
from __future__ import annotations

import zlib

import numpy as np

# Model dimensions (Diffusers release blog for FLUX.3 Image Klein, "Speed,
# architecture, and how the tokens move"; Klein local-run guide, "Inside the
# transformer").
DIM = 3072
HEADS = 24
HEAD_DIM = 128
MLP_HIDDEN = 9216
LATENT_CH = 128
TIME_FREQ_DIM = 256
N_STAGE1 = 5
N_JOINT = 28
MODES = ("txt", "img", "ref")

WEIGHT_SEED = 0
INPUT_SEED = 1
NOISE_SEED = 2


def round_to_bf16(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even), as float32."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    bias = 0x7FFF + ((u >> 16) & 1)
    r = ((u + bias) & 0xFFFF0000).astype(np.uint32)
    return r.view(np.float32).reshape(a.shape)


def _rng(seed: int, tag: str) -> np.random.Generator:
    key = zlib.crc32(tag.encode("utf-8"))
    return np.random.default_rng(np.random.SeedSequence([int(seed), key]))


def normal(seed: int, tag: str, shape, std: float = 1.0, mean: float = 0.0,
           bf16: bool = True) -> np.ndarray:
    """float32 array of N(mean, std^2) draws keyed by (seed, tag)."""
    g = _rng(seed, tag)
    a = g.standard_normal(size=tuple(shape), dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    if mean != 0.0:
        a += np.float32(mean)
    return round_to_bf16(a) if bf16 else a


def linear(seed: int, tag: str, n_out: int, n_in: int) -> np.ndarray:
    return normal(seed, tag, (n_out, n_in), std=1.0 / np.sqrt(n_in))


# ---------------------------------------------------------------------------
# Weights
# ---------------------------------------------------------------------------

def block_weights(seed: int, name: str) -> dict:
    """One block's weights.

    w_in  [3*DIM + 2*MLP_HIDDEN, DIM]: rows q | k | v | gate | up.
    w_out [DIM, DIM + MLP_HIDDEN]:     columns attn-out | mlp-down.
    q_norm, k_norm [HEAD_DIM].
    """
    w_in = linear(seed, f"{name}.w_in", 3 * DIM + 2 * MLP_HIDDEN, DIM)
    w_o = linear(seed, f"{name}.w_attn_out", DIM, DIM)
    w_d = linear(seed, f"{name}.w_mlp_down", DIM, MLP_HIDDEN)
    w_out = np.concatenate([w_o, w_d], axis=1)
    q_norm = normal(seed, f"{name}.q_norm", (HEAD_DIM,), std=0.1, mean=1.0, bf16=False)
    k_norm = normal(seed, f"{name}.k_norm", (HEAD_DIM,), std=0.1, mean=1.0, bf16=False)
    return {"w_in": w_in, "w_out": np.ascontiguousarray(w_out),
            "q_norm": q_norm, "k_norm": k_norm}


def block_name(stage: int, mode: str | None, index: int) -> str:
    if stage == 1:
        return f"stage1.{mode}.{index}"
    return f"joint.{index}"


TEXT_STACK = 8 * 2560  # eight encoder layers of width 2560, stacked per text token


def misc_weights(seed: int, distilled: bool, txt_in: bool = False) -> dict:
    """Everything that is not a block: embedders, modulation, in/out layers
    (txt_in: also the 20480 -> 3072 text input projection)."""
    w = {
        "img_in": linear(seed, "img_in", DIM, LATENT_CH),
        "ref_in": linear(seed, "ref_in", DIM, LATENT_CH),
        "t_mlp1": linear(seed, "t_mlp1", DIM, TIME_FREQ_DIM),
        "t_mlp2": linear(seed, "t_mlp2", DIM, DIM),
        "final_mod": linear(seed, "final_mod", 2 * DIM, DIM),
        "final_out": linear(seed, "final_out", LATENT_CH, DIM),
    }
    for stage in (1, 2):
        for m in MODES:
            w[f"mod{stage}.{m}"] = linear(seed, f"mod{stage}.{m}", 3 * DIM, DIM)
    if distilled:
        w["tt_mlp1"] = linear(seed, "tt_mlp1", DIM, TIME_FREQ_DIM)
        w["tt_mlp2"] = linear(seed, "tt_mlp2", DIM, DIM)
    if txt_in:
        w["txt_in"] = linear(seed, "txt_in", DIM, TEXT_STACK)
    return w


class ModelWeights:
    """Lazily generated, cached random-init weights for a whole stack.

    n_stage1 / n_joint default to the model's 5 and 28; tests may ask for
    fewer blocks to exercise the orchestration cheaply.
    """

    def __init__(self, seed: int = WEIGHT_SEED, distilled: bool = True,
                 n_stage1: int = N_STAGE1, n_joint: int = N_JOINT, txt_in: bool = False):
        self.seed = seed
        self.distilled = distilled
        self.n_stage1 = n_stage1
        self.n_joint = n_joint
        self.txt_in = txt_in
        self._blocks: dict = {}
        self._misc = None

    @property
    def misc(self) -> dict:
        if self._misc is None:
            self._misc = misc_weights(self.seed, self.distilled, self.txt_in)
        return self._misc

    def block(self, stage: int, mode: str | None, index: int) -> dict:
        key = block_name(stage, mode, index)
        if key not in self._blocks:
            self._blocks[key] = block_weights(self.seed, key)
        return self._blocks[key]

    def stage1(self, mode: str) -> list:
        return [self.block(1, mode, i) for i in range(self.n_stage1)]

    def joint(self) -> list:
        return [self.block(2, None, i) for i in range(self.n_joint)]


# ---------------------------------------------------------------------------
# Activations
# ---------------------------------------------------------------------------

def tokens(seed: int, tag: str, batch: int, rows: int) -> np.ndarray:
    """Residual-stream tokens [batch, rows, DIM], N(0,1), bf16-representable."""
    return normal(seed, f"tokens.{tag}", (batch, rows, DIM))


def text_embeddings(seed: int, batch: int, n_txt: int) -> np.ndarray:
    """Text-encoder output stand-in [batch, n_txt, DIM]; batch 2 = cond, uncond."""
    return normal(seed, "text_emb", (batch, n_txt, DIM))


def text_hidden_states(seed: int, batch: int, n_txt: int) -> np.ndarray:
    """Stacked text-encoder hidden states stand-in [batch, n_txt, 20480], N(0,1)."""
    return normal(seed, "text_hidden", (batch, n_txt, TEXT_STACK))


def noise_latents(seed: int, n_img: int) -> np.ndarray:
    """Packed noise latents [n_img, 128] (float32, not rounded)."""
    return normal(seed, "noise", (n_img, LATENT_CH), bf16=False)


def ref_latents(seed: int, n_ref: int) -> np.ndarray:
    """Packed reference latents [n_ref, 128] (float32, not rounded)."""
    return normal(seed, "ref_latents", (n_ref, LATENT_CH), bf16=False)


def modulation_vectors(seed: int, tag: str, n_modes: int = 3) -> np.ndarray:
    """Stand-in modulation [n_modes, 3 (shift, scale, gate), DIM], N(0, 0.5^2)."""
    return normal(seed, f"mod.{tag}", (n_modes, 3, DIM), std=0.5, bf16=False)


def velocity(seed: int, tag: str, batch: int, n_img: int) -> np.ndarray:
    return normal(seed, f"velocity.{tag}", (batch, n_img, LATENT_CH), bf16=False)
