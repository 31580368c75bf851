"""Python binding of the Klein C-ABI library (include/klein.h).

Argument marshalling only: every step of the denoiser runs in the CUDA
kernels of libklein.so. Tensors are torch CUDA tensors (device memory and
streams come from PyTorch); each function passes their data pointers and the
current CUDA stream to the C function of the same name and raises
KleinError on a negative status. There is no CPU fallback: importing this
module fails if the library is missing.
"""
from __future__ import annotations

import ctypes
import os

from ctypes import POINTER, Structure, c_float, c_int, c_longlong, c_size_t, c_uint, c_ulonglong, c_void_p

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.environ.get("KLEIN_LIB") or os.path.join(HERE, "lib", "libklein.so")

DIM = 3072
HEADS = 24
HEAD_DIM = 128
MLP_HIDDEN = 9216
LATENT_CH = 128
MAX_REFS = 10
IN_COLS = 3 * DIM + 2 * MLP_HIDDEN
OUT_K = DIM + MLP_HIDDEN

STATUS = {0: "KLEIN_OK", -1: "KLEIN_ERR_INVALID_ARG", -2: "KLEIN_ERR_SHAPE", -3: "KLEIN_ERR_ALIGN",
          -4: "KLEIN_ERR_WORKSPACE", -5: "KLEIN_ERR_CUDA", -6: "KLEIN_ERR_TIMEOUT", -7: "KLEIN_ERR_UNSUPPORTED"}


class KleinError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{STATUS.get(code, code)}: {msg}")
        self.code = code
        self.name = STATUS.get(code, str(code))


if not os.path.exists(LIB_PATH):
    raise ImportError(f"libklein.so not built ({LIB_PATH}); run `python -m latent_flow_matching_joint_b200.build`")
lib = ctypes.CDLL(LIB_PATH)


class KleinSeq(Structure):
    _fields_ = [("batch", c_int), ("n_txt", c_int), ("img_h", c_int), ("img_w", c_int), ("n_refs", c_int),
                ("ref_h", c_int * MAX_REFS), ("ref_w", c_int * MAX_REFS)]


class KleinBlockWeights(Structure):
    _fields_ = [("w_in", c_void_p), ("w_out", c_void_p), ("q_norm", c_void_p), ("k_norm", c_void_p),
                ("w_in_scale", c_void_p), ("w_out_scale", c_void_p), ("w_in_sf", c_void_p), ("w_out_sf", c_void_p)]


NVFP4_MATRIX, NVFP4_ROWS, NVFP4_IN_PROJ = 0, 1, 2


class KleinModelDesc(Structure):
    _fields_ = [("n_stage1", c_int), ("n_joint", c_int), ("stage1", c_void_p * 3), ("joint", c_void_p),
                ("img_in", c_void_p), ("ref_in", c_void_p), ("t_mlp1", c_void_p), ("t_mlp2", c_void_p),
                ("tt_mlp1", c_void_p), ("tt_mlp2", c_void_p), ("mod", (c_void_p * 3) * 2),
                ("final_mod", c_void_p), ("final_out", c_void_p), ("txt_in", c_void_p)]


_SIGS = {
    "klein_last_error": (ctypes.c_char_p, []),
    "klein_version": (c_int, []),
    "klein_launch_count": (c_longlong, []),
    "klein_device_status": (c_int, [POINTER(c_uint)]),
    "klein_sync": (c_int, [c_void_p]),
    "klein_set_wait_limit_ns": (c_int, [c_ulonglong]),
    "klein_wait_probe": (c_int, [c_ulonglong, c_void_p]),
    "klein_profile_begin": (c_int, [c_int]),
    "klein_profile_end": (c_int, [POINTER(ctypes.c_double), POINTER(c_int)]),
    "klein_seq_tokens": (c_int, [POINTER(KleinSeq), POINTER(c_int), POINTER(c_int), POINTER(c_int)]),
    "klein_pad_text_len": (c_int, [c_int]),
    "klein_sigma_schedule": (c_int, [c_int, c_float, POINTER(c_float)]),
    "klein_positions": (c_int, [POINTER(KleinSeq), c_void_p, c_void_p]),
    "klein_block_workspace_size": (c_size_t, [c_int, c_int]),
    "klein_block_forward": (c_int, [POINTER(KleinBlockWeights), c_void_p, c_int, c_int, c_int, c_int, c_int, c_int,
                                    c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "klein_block_forward_static": (c_int, [POINTER(KleinBlockWeights), c_void_p, c_int, c_int, c_int, c_int, c_int,
                                           c_int, c_void_p, c_void_p, c_void_p]),
    "klein_model_create": (c_int, [POINTER(c_void_p), POINTER(KleinModelDesc)]),
    "klein_model_destroy": (None, [c_void_p]),
    "klein_stack_workspace_size": (c_size_t, [POINTER(KleinSeq)]),
    "klein_stack_forward": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_float, c_float, POINTER(KleinSeq),
                                    c_void_p, c_void_p, c_size_t, c_void_p]),
    "klein_denoise": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_float, c_float, POINTER(KleinSeq),
                              c_void_p, c_int, c_void_p, c_size_t, c_void_p]),
    "klein_op_modln": (c_int, [c_void_p, c_int, c_int, c_int, c_int, c_int, c_int, c_void_p, c_longlong, c_int,
                               c_void_p, c_void_p]),
    "klein_op_rope_table": (c_int, [c_void_p, c_int, c_float, c_void_p, c_void_p]),
    "klein_op_rope": (c_int, [c_void_p, c_void_p, c_void_p, c_int, c_int, c_void_p]),
    "klein_op_euler": (c_int, [c_void_p, c_void_p, c_void_p, c_longlong, c_float, c_float, c_void_p, c_float,
                               c_void_p]),
    "klein_op_gemm": (c_int, [c_void_p, c_void_p, c_void_p, c_int, c_int, c_int, c_void_p]),
    "klein_op_gemm_e4m3": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_int, c_int,
                                   c_void_p]),
    "klein_op_modln_e4m3": (c_int, [c_void_p, c_int, c_int, c_int, c_int, c_int, c_int, c_void_p, c_longlong,
                                    c_void_p, c_void_p, c_void_p]),
    "klein_quantize_rowwise_e4m3": (c_int, [c_void_p, c_longlong, c_int, c_void_p, c_void_p, c_void_p]),
    "klein_op_attention": (c_int, [c_void_p, c_void_p, c_void_p, c_int, c_int, c_int, c_void_p, c_longlong,
                                   c_void_p]),
    "klein_quantize_nvfp4": (c_int, [c_void_p, c_longlong, c_int, c_int, c_void_p, c_void_p, c_void_p, c_void_p]),
    "klein_op_modln_nvfp4": (c_int, [c_void_p, c_int, c_int, c_int, c_int, c_int, c_int, c_void_p, c_longlong,
                                     c_void_p, c_void_p, c_void_p, c_void_p]),
    "klein_op_gemm_nvfp4": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_int,
                                    c_int, c_void_p]),
    "klein_op_time_mod": (c_int, [c_void_p, c_float, c_float, c_int, c_void_p, c_void_p, c_void_p, c_size_t,
                                  c_void_p]),
}

for _name, (_res, _args) in _SIGS.items():
    _f = getattr(lib, _name)
    _f.restype = _res
    _f.argtypes = _args

EXPORTED = tuple(_SIGS)


def _check(rc: int) -> int:
    if rc < 0:
        raise KleinError(rc, lib.klein_last_error().decode(errors="replace"))
    return rc


def _ptr(t):
    return None if t is None else c_void_p(t.data_ptr())


def _stream(stream):
    if stream is not None:
        return c_void_p(stream)
    import torch
    return c_void_p(torch.cuda.current_stream().cuda_stream)


def make_seq(batch: int, n_txt: int, img_h: int, img_w: int, refs=()) -> KleinSeq:
    s = KleinSeq()
    s.batch, s.n_txt, s.img_h, s.img_w, s.n_refs = batch, n_txt, img_h, img_w, len(refs)
    for k, (h, w) in enumerate(refs):
        s.ref_h[k], s.ref_w[k] = h, w
    return s


# ------------------------------------------------------------------ host helpers

def klein_version() -> int:
    return lib.klein_version()


def klein_launch_count() -> int:
    return lib.klein_launch_count()


def klein_pad_text_len(n: int) -> int:
    return lib.klein_pad_text_len(n)


def klein_sigma_schedule(steps: int, shift: float = 6.93):
    out = (c_float * (steps + 1))()
    _check(lib.klein_sigma_schedule(steps, shift, out))
    return list(out)


def klein_seq_tokens(seq: KleinSeq):
    ni, nr, nt = c_int(), c_int(), c_int()
    _check(lib.klein_seq_tokens(ctypes.byref(seq), ctypes.byref(ni), ctypes.byref(nr), ctypes.byref(nt)))
    return ni.value, nr.value, nt.value


def klein_device_status():
    site = c_uint()
    rc = lib.klein_device_status(ctypes.byref(site))
    return rc, site.value, lib.klein_last_error().decode(errors="replace")


def klein_sync(stream=None):
    """(status, message) after the stream's queued work: 0, or KLEIN_ERR_TIMEOUT
    when a bounded device wait gave up (read and cleared)."""
    rc = lib.klein_sync(_stream(stream))
    return rc, lib.klein_last_error().decode(errors="replace")


def klein_set_wait_limit_ns(ns: int):
    _check(lib.klein_set_wait_limit_ns(ns))


def klein_wait_probe(limit_ns: int, stream=None):
    _check(lib.klein_wait_probe(limit_ns, _stream(stream)))


PROF_KINDS = ("modln", "gemm_in", "attention", "gemm_out", "time_mod", "projections", "euler", "other", "quant",
              "modln_s1", "gemm_in_s1", "attention_s1", "gemm_out_s1")


def klein_profile_begin(max_launches: int):
    _check(lib.klein_profile_begin(max_launches))


def klein_profile_end():
    """-> {kind: (total_ms, launches)} for the launches since klein_profile_begin."""
    ms = (ctypes.c_double * len(PROF_KINDS))()
    n = (c_int * len(PROF_KINDS))()
    _check(lib.klein_profile_end(ms, n))
    return {k: (ms[i], n[i]) for i, k in enumerate(PROF_KINDS)}


def klein_block_workspace_size(batch: int, rows: int) -> int:
    return lib.klein_block_workspace_size(batch, rows)


def klein_stack_workspace_size(seq: KleinSeq) -> int:
    return lib.klein_stack_workspace_size(ctypes.byref(seq))


# ------------------------------------------------------------------ device calls

def klein_positions(seq: KleinSeq, pos, stream=None):
    _check(lib.klein_positions(ctypes.byref(seq), _ptr(pos), _stream(stream)))


def block_weights(w: dict) -> KleinBlockWeights:
    """KleinBlockWeights from a dict of CUDA tensors w_in, w_out, q_norm, k_norm
    (+ w_in_scale, w_out_scale for a rowwise FP8 block, see quantize_block_e4m3;
    + w_in_sf, w_out_sf for an NVFP4 block, see quantize_block_nvfp4)."""
    def p(name):
        t = w.get(name)
        return t.data_ptr() if t is not None else None
    return KleinBlockWeights(p("w_in"), p("w_out"), p("q_norm"), p("k_norm"), p("w_in_scale"), p("w_out_scale"),
                             p("w_in_sf"), p("w_out_sf"))


def klein_quantize_rowwise_e4m3(src, codes, scale, stream=None):
    """Rowwise e4m3 codes (uint8, same shape) and scales (float32 [rows]) of a
    bf16 [rows, cols] CUDA tensor."""
    rows, cols = src.shape
    _check(lib.klein_quantize_rowwise_e4m3(_ptr(src), rows, cols, _ptr(codes), _ptr(scale), _stream(stream)))


def quantize_block_e4m3(w: dict, stream=None) -> dict:
    """A rowwise FP8 copy of one block's bf16 weights (new device tensors)."""
    import torch
    out = {"q_norm": w["q_norm"], "k_norm": w["k_norm"]}
    for name in ("w_in", "w_out"):
        src = w[name]
        codes = torch.empty(src.shape, dtype=torch.uint8, device=src.device)
        scale = torch.empty(src.shape[0], dtype=torch.float32, device=src.device)
        klein_quantize_rowwise_e4m3(src, codes, scale, stream)
        out[name], out[name + "_scale"] = codes, scale
    return out


def nvfp4_scale_bytes(rows: int, cols: int, mode: int) -> int:
    """Bytes of the block-scale atoms klein_quantize_nvfp4 writes."""
    pad = 256 if mode == NVFP4_ROWS else 128
    return (rows + pad - 1) // pad * pad * cols // 16


def klein_quantize_nvfp4(src, mode: int, stream=None):
    """NVFP4 codes (uint8 [rows, cols/2]), block scales (uint8 atoms) and
    second-level scales (float32 [1] or [rows]) of a bf16 [rows, cols] CUDA
    tensor (new device tensors)."""
    import torch
    rows, cols = src.shape
    codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=src.device)
    sf = torch.empty(nvfp4_scale_bytes(rows, cols, mode), dtype=torch.uint8, device=src.device)
    g = torch.empty(rows if mode == NVFP4_ROWS else 4, dtype=torch.float32, device=src.device)
    _check(lib.klein_quantize_nvfp4(_ptr(src), rows, cols, mode, _ptr(codes), _ptr(sf), _ptr(g), _stream(stream)))
    return codes, sf, g


def quantize_block_nvfp4(w: dict, stream=None) -> dict:
    """An NVFP4 copy of one block's bf16 weights (new device tensors); w_in
    in the in-projection's NVFP4 row order."""
    out = {"q_norm": w["q_norm"], "k_norm": w["k_norm"]}
    for name, mode in (("w_in", NVFP4_IN_PROJ), ("w_out", NVFP4_MATRIX)):
        codes, sf, g = klein_quantize_nvfp4(w[name], mode, stream)
        out[name], out[name + "_sf"], out[name + "_scale"] = codes, sf, g
    return out


def klein_op_modln_nvfp4(x, row0: int, rows: int, n_txt: int, n_img: int, mod, codes, sf, g, stream=None):
    batch, n_total = x.shape[0], x.shape[1]
    stride = mod.shape[-2] * mod.shape[-1]
    _check(lib.klein_op_modln_nvfp4(_ptr(x), batch, n_total, row0, rows, n_txt, n_img, _ptr(mod), stride, _ptr(codes),
                                    _ptr(sf), _ptr(g), _stream(stream)))


def klein_op_gemm_nvfp4(a, a_sf, a_g, b, b_sf, b_g, c, stream=None):
    m, kh = a.shape
    n = b.shape[0]
    _check(lib.klein_op_gemm_nvfp4(_ptr(a), _ptr(a_sf), _ptr(a_g), _ptr(b), _ptr(b_sf), _ptr(b_g), _ptr(c), m, n,
                                   2 * kh, _stream(stream)))


def klein_block_forward(w: dict, x, n_txt: int, n_img: int, pos, mod, ws, row0: int = 0, rows: int | None = None,
                        stream=None):
    batch, n_total = x.shape[0], x.shape[1]
    rows = n_total - row0 if rows is None else rows
    bw = block_weights(w)
    _check(lib.klein_block_forward(ctypes.byref(bw), _ptr(x), batch, n_total, row0, rows, n_txt, n_img, _ptr(pos),
                                   _ptr(mod), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))


def klein_block_forward_static(w: dict, x, n_txt: int, n_img: int, pos, mod, row0: int = 0,
                               rows: int | None = None, stream=None):
    """klein_block_forward with the library's fixed scratch instead of a
    workspace (for callers that cannot allocate); batch * rows <= 256."""
    batch, n_total = x.shape[0], x.shape[1]
    rows = n_total - row0 if rows is None else rows
    bw = block_weights(w)
    _check(lib.klein_block_forward_static(ctypes.byref(bw), _ptr(x), batch, n_total, row0, rows, n_txt, n_img,
                                          _ptr(pos), _ptr(mod), _stream(stream)))


class KleinModel:
    """A klein_model handle over device tensors (the tensors stay owned here).

    tensors: dict with "stage1": {mode: [block dict]*n}, "joint": [block dict],
    and the misc weights img_in, ref_in, t_mlp1, t_mlp2, tt_mlp1, tt_mlp2,
    "mod1.txt" ... "mod2.ref", final_mod, final_out (bf16 [out, in]).
    """

    MODES = ("txt", "img", "ref")

    def __init__(self, tensors: dict):
        self.tensors = tensors
        st1 = tensors["stage1"]
        n1 = len(st1["txt"])
        joint = tensors["joint"]
        self._st1 = []
        d = KleinModelDesc()
        d.n_stage1, d.n_joint = n1, len(joint)
        for i, m in enumerate(self.MODES):
            blocks = st1.get(m) or []
            arr = (KleinBlockWeights * max(1, len(blocks)))(*[block_weights(b) for b in blocks])
            self._st1.append(arr)
            d.stage1[i] = ctypes.cast(arr, c_void_p) if blocks else None
        self._joint = (KleinBlockWeights * max(1, len(joint)))(*[block_weights(b) for b in joint])
        d.joint = ctypes.cast(self._joint, c_void_p) if joint else None
        g = tensors.get
        for name in ("img_in", "ref_in", "t_mlp1", "t_mlp2", "tt_mlp1", "tt_mlp2", "final_mod", "final_out",
                     "txt_in"):
            t = g(name)
            setattr(d, name, t.data_ptr() if t is not None else None)
        for s in (0, 1):
            for i, m in enumerate(self.MODES):
                t = g(f"mod{s + 1}.{m}")
                d.mod[s][i] = t.data_ptr() if t is not None else None
        self.desc = d
        self.distilled = g("tt_mlp1") is not None
        h = c_void_p()
        _check(lib.klein_model_create(ctypes.byref(h), ctypes.byref(d)))
        self.handle = h

    def __del__(self):
        h = getattr(self, "handle", None)
        if h is not None and h.value:
            lib.klein_model_destroy(h)
            self.handle = None


def klein_stack_forward(model: KleinModel, latents, text, refs, sigma: float, sigma_next: float, seq: KleinSeq,
                        v_out, ws, stream=None):
    _check(lib.klein_stack_forward(model.handle, _ptr(latents), _ptr(text), _ptr(refs), sigma, sigma_next,
                                   ctypes.byref(seq), _ptr(v_out), _ptr(ws), ws.numel() * ws.element_size(),
                                   _stream(stream)))


def klein_denoise(model: KleinModel, latents, text, refs, steps: int, cfg: float, seq: KleinSeq, ws,
                  shift: float = 6.93, x0_out=None, x0_every_step: bool = False, stream=None):
    _check(lib.klein_denoise(model.handle, _ptr(latents), _ptr(text), _ptr(refs), steps, cfg, shift,
                             ctypes.byref(seq), _ptr(x0_out), int(x0_every_step), _ptr(ws),
                             ws.numel() * ws.element_size(), _stream(stream)))


def klein_op_modln(x, row0: int, rows: int, n_txt: int, n_img: int, mod, h, single_mode: bool = False,
                   mod_stride: int | None = None, stream=None):
    batch, n_total = x.shape[0], x.shape[1]
    stride = mod_stride if mod_stride is not None else (mod.shape[-2] * mod.shape[-1] if mod.dim() == 3 else 0)
    _check(lib.klein_op_modln(_ptr(x), batch, n_total, row0, rows, n_txt, n_img, _ptr(mod), stride,
                              int(single_mode), _ptr(h), _stream(stream)))


def klein_op_rope_table(pos, table, theta: float = 10000.0, stream=None):
    _check(lib.klein_op_rope_table(_ptr(pos), pos.shape[0], theta, _ptr(table), _stream(stream)))


def klein_op_rope(inp, out, table, stream=None):
    rows, heads = inp.shape[0], inp.shape[1]
    _check(lib.klein_op_rope(_ptr(inp), _ptr(out), _ptr(table), rows, heads, _stream(stream)))


def klein_op_euler(x, v_cond, v_uncond, dsigma: float, g: float = 1.0, x0_out=None, sigma: float = 0.0,
                   stream=None):
    _check(lib.klein_op_euler(_ptr(x), _ptr(v_cond), _ptr(v_uncond), x.numel(), dsigma, g, _ptr(x0_out), sigma,
                              _stream(stream)))


def klein_op_gemm(a, b, c, stream=None):
    m, k = a.shape
    n = b.shape[0]
    _check(lib.klein_op_gemm(_ptr(a), _ptr(b), _ptr(c), m, n, k, _stream(stream)))


def klein_op_gemm_e4m3(a, a_scale, b, b_scale, c, stream=None):
    m, k = a.shape
    n = b.shape[0]
    _check(lib.klein_op_gemm_e4m3(_ptr(a), _ptr(a_scale), _ptr(b), _ptr(b_scale), _ptr(c), m, n, k,
                                  _stream(stream)))


def klein_op_modln_e4m3(x, row0: int, rows: int, n_txt: int, n_img: int, mod, codes, scale, stream=None):
    batch, n_total = x.shape[0], x.shape[1]
    stride = mod.shape[-2] * mod.shape[-1]
    _check(lib.klein_op_modln_e4m3(_ptr(x), batch, n_total, row0, rows, n_txt, n_img, _ptr(mod), stride,
                                   _ptr(codes), _ptr(scale), _stream(stream)))


def klein_op_attention(q, k, vt, rows: int, out, stream=None):
    batch, rows_pad = q.shape[0], q.shape[2]
    _check(lib.klein_op_attention(_ptr(q), _ptr(k), _ptr(vt), batch, rows, rows_pad, _ptr(out), out.shape[-1],
                                  _stream(stream)))


def klein_op_time_mod(model: KleinModel, sigma: float, sigma_next: float, with_ref: bool, mod_out, final_out, ws,
                      stream=None):
    _check(lib.klein_op_time_mod(model.handle, sigma, sigma_next, int(with_ref), _ptr(mod_out), _ptr(final_out),
                                 _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))
