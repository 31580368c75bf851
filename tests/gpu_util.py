"""Helpers for the GPU parity tests: upload seeded inputs, compare results."""
import numpy as np
import torch

import klein_inputs as ki


def dev():
    return torch.device("cuda:0")


def to_bf16(a: np.ndarray) -> torch.Tensor:
    """bf16-representable float32 array -> bf16 CUDA tensor (exact)."""
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(dev()).to(torch.bfloat16)


def to_f32(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(dev())


def host(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def upload_block(w: dict) -> dict:
    return {"w_in": to_bf16(w["w_in"]), "w_out": to_bf16(w["w_out"]),
            "q_norm": to_f32(w["q_norm"]), "k_norm": to_f32(w["k_norm"])}


def upload_model(m: ki.ModelWeights, with_ref: bool = True) -> dict:
    t = {"stage1": {}, "joint": [upload_block(b) for b in m.joint()]}
    for mode in ki.MODES:
        if mode == "ref" and not with_ref:
            t["stage1"][mode] = []
            continue
        t["stage1"][mode] = [upload_block(b) for b in m.stage1(mode)]
    for k, v in m.misc.items():
        t[k] = to_bf16(v)
    return t


def workspace(nbytes: int) -> torch.Tensor:
    return torch.empty(nbytes, dtype=torch.uint8, device=dev())


def rms(a) -> float:
    return float(np.sqrt(np.mean(np.square(a))))


def max_err_ratio(got, ref) -> float:
    """max |got - ref| / RMS(ref): the block tolerance metric (<= 2e-2)."""
    return float(np.max(np.abs(got - ref)) / rms(ref))


def cosine(a, b) -> float:
    a = np.ravel(a)
    b = np.ravel(b)
    return float(a @ b / (np.linalg.norm(a) * np.linalg.norm(b)))
