"""Writes the oracle's outputs at the full model size and the benchmarked
sequence lengths, for the GPU parity tests in tests/test_gpu_full_size.py.

Model: random-init 5 + 28 block distilled stack (klein_inputs weights, seed
0). Inputs: text embeddings seed 1, noise seed 2, reference latents seed 1.
Cases (each written once; an existing file is kept):

  stack_t2i_1024   one denoiser call (the first Euler step: sigma = 1,
                   sigma_next = the second level of the 16-step schedule) at
                   512 text + 64x64 image tokens: velocity [1, 4096, 128]
  stack_edit_1024  the same call with one 64x64 reference (512 + 4096 + 4096
                   tokens): velocity [1, 4096, 128]
  denoise_t2i_1024 the full 16-step shifted Euler denoise at 512 + 64x64
                   tokens: final latents [4096, 128]
  stack_t2i4k_rows one call of a 0 + 1 block stack (the first joint block of
                   the same model, no stage 1) at the largest output, 4096 x
                   4096: 512 text + 256 x 256 image tokens (66048); the
                   velocity of a sample of image rows [1, rows, 128], the row
                   indices stored beside it

Calls only the oracle and the seeded input generators; a float64 run of
tens of TFLOP per denoiser call, so this takes hours on a few host cores.

    python tests/golden/make_full_size_goldens.py [case ...]
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

HERE = os.path.dirname(os.path.abspath(__file__))
N_TXT, GRID, STEPS = 512, (64, 64), 16
CASES = {
    # name: (references, kind)
    "stack_t2i_1024": ((), "stack"),
    "stack_edit_1024": (((64, 64),), "stack"),
    "denoise_t2i_1024": ((), "denoise"),
    "stack_t2i4k_rows": ((), "stack_rows"),
}
GRID_4K = (256, 256)


def sample_rows_4k():
    """Image rows of the 4096x4096 case: every 1021st token plus the grid's
    corners and the middle of its first and last rows."""
    n = GRID_4K[0] * GRID_4K[1]
    extra = [0, GRID_4K[1] - 1, GRID_4K[1] // 2, n // 2, n - GRID_4K[1], n - 1]
    return np.unique(np.concatenate([np.arange(0, n, 1021), extra]))


def path_of(name):
    return os.path.join(HERE, name + ".npy")


def run(name, model):
    refs, kind = CASES[name]
    t0 = time.time()
    grid = GRID_4K if kind == "stack_rows" else GRID
    n_img = grid[0] * grid[1]
    n_ref = sum(h * w for h, w in refs)
    text = ki.text_embeddings(ki.INPUT_SEED, 1, N_TXT)
    noise = ki.noise_latents(ki.NOISE_SEED, n_img)
    rl = ki.ref_latents(ki.INPUT_SEED, n_ref) if n_ref else None
    pos = o.positions(N_TXT, grid, refs)
    sig = o.sigma_schedule(STEPS)
    meta = {"n_txt": N_TXT, "grid": grid, "refs": refs, "steps": STEPS, "distilled": True,
            "weight_seed": ki.WEIGHT_SEED, "text_seed": ki.INPUT_SEED, "noise_seed": ki.NOISE_SEED,
            "ref_seed": ki.INPUT_SEED, "kind": kind, "n_stage1": model.n_stage1, "n_joint": model.n_joint}
    if kind == "stack":
        out = o.transformer(model, noise, text, rl, pos, sig[0], sig[1])
        meta.update({"sigma": float(sig[0]), "sigma_next": float(sig[1])})
    elif kind == "stack_rows":
        rows = sample_rows_4k()
        out = o.transformer(model, noise, text, rl, pos, sig[0], sig[1], img_rows=rows)
        meta.update({"sigma": float(sig[0]), "sigma_next": float(sig[1]), "img_rows": rows.tolist()})
    else:
        def on_step(i, x, v, s):
            print(f"  {name}: step {i + 1}/{STEPS} done after {time.time() - t0:.0f} s", flush=True)
        out = o.denoise(model, noise, text, rl, pos, STEPS, on_step=on_step)
    np.save(path_of(name), np.asarray(out, dtype=np.float32))
    meta["seconds"] = round(time.time() - t0, 1)
    meta["dtype"] = "float32 (oracle float64, rounded once)"
    with open(path_of(name).replace(".npy", ".json"), "w") as f:
        json.dump(meta, f, indent=1)
    print(name, meta, flush=True)


def main(names):
    model = ki.ModelWeights(seed=ki.WEIGHT_SEED, distilled=True)
    for name in names or list(CASES):
        if os.path.exists(path_of(name)):
            print(name, "exists; kept", flush=True)
            continue
        if CASES[name][1] == "stack_rows":
            run(name, ki.ModelWeights(seed=ki.WEIGHT_SEED, distilled=True, n_stage1=0, n_joint=1))
        else:
            run(name, model)


if __name__ == "__main__":
    main(sys.argv[1:])
