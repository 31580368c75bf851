"""Writes the oracle's final latents of a full-depth distilled denoise.

Model: random-init 5 + 28 block distilled stack (klein_inputs weights, seed 0).
Sequence: 80 text tokens (text seed 1) + 8 x 8 image tokens, batch 1, no
reference; noise seed 2; 16 shifted Euler steps (shift 6.93). Calls only the
oracle and the seeded input generators; the GPU test compares its own
full-depth denoise of the same inputs against this file.

    python tests/golden/make_denoise_golden.py
"""
import json
import os
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import klein_inputs as ki  # noqa: E402
import oracle as o  # noqa: E402

N_TXT, GRID, STEPS = 80, (8, 8), 16
OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "denoise_full_depth_80_8x8_16.npy")


def main():
    t0 = time.time()
    m = ki.ModelWeights(seed=ki.WEIGHT_SEED, distilled=True)
    text = ki.text_embeddings(ki.INPUT_SEED, 1, N_TXT)
    noise = ki.noise_latents(ki.NOISE_SEED, GRID[0] * GRID[1])
    x = o.denoise(m, noise, text, None, o.positions(N_TXT, GRID), STEPS)
    np.save(OUT, x.astype(np.float64))
    meta = {"n_txt": N_TXT, "grid": GRID, "steps": STEPS, "distilled": True, "weight_seed": ki.WEIGHT_SEED,
            "text_seed": ki.INPUT_SEED, "noise_seed": ki.NOISE_SEED, "seconds": round(time.time() - t0, 1)}
    with open(OUT.replace(".npy", ".json"), "w") as f:
        json.dump(meta, f, indent=1)
    print(OUT, meta)


if __name__ == "__main__":
    main()
