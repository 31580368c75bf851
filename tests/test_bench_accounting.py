"""The benchmark's work accounting, against counts written out by hand.

The bench reports the method's FLOPs per denoise step and the FLOPs the
library actually executes (the image and reference streams' stage 1 shared by
the batch items; the base model's text and reference stage 1 computed at the
first step only), and times the in-projection over the rows it really
processes. These checks recount both for the three workloads."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

D, F = 3072, 9216


def _block(rows):
    # QKV + MLP-in (D x (3D + 2F)), out-projection ((D + F) x D), attention 4 N^2 D
    return rows * (2 * D * (3 * D + 2 * F) + 2 * (D + F) * D) + 4.0 * rows * rows * D


def test_block_flops_per_token():
    assert bench.block_gemm_flops_per_token() == 2 * D * (3 * D + 2 * F) + 2 * (D + F) * D
    # the 512 + 4096 joint block: 1.3916 TFLOP
    assert abs(_block(4608) / 1e12 - 1.3916) < 1e-4


def test_method_flops_per_step():
    # t2i: stage 1 text (512) and image (4096), 28 joint blocks over 4608, projections
    f = 5 * (_block(512) + _block(4096)) + 28 * _block(4608) + 2.0 * 4096 * 128 * D * 2
    assert abs(bench.step_flops(1, 512, 4096, 0) - f) < 1e-6 * f
    assert abs(f / 1e12 - 45.67) < 0.01


def test_executed_flops_distilled_equals_method():
    for batch, n_txt, n_img, n_ref in ((1, 512, 4096, 0), (1, 512, 4096, 4096)):
        ex = bench.executed_denoise_flops(batch, n_txt, n_img, n_ref, 16, True)
        assert abs(ex - 16 * bench.step_flops(batch, n_txt, n_img, n_ref)) < 1e-9 * ex


def test_executed_flops_base_model_cfg():
    # 2048x2048 under guidance: batch 2, 50 steps. The image stream's stage 1
    # runs once per step for both items; the text stream's stage 1 (both
    # items) runs at the first step only; the joint blocks and the output
    # layer run per item every step.
    steps, n_txt, n_img = 50, 560, 16384
    n = n_txt + n_img
    expect = (5 * 2 * _block(n_txt) + steps * 5 * _block(n_img) + steps * 2 * 28 * _block(n)
              + steps * 2.0 * n_img * 128 * D + steps * 2 * 2.0 * n_img * D * 128)
    got = bench.executed_denoise_flops(2, n_txt, n_img, 0, steps, False)
    assert abs(got - expect) < 1e-9 * expect
    method = steps * bench.step_flops(2, n_txt, n_img, 0)
    assert 0.90 < got / method < 0.95


def test_in_projection_rows():
    # t2i: per step 5 x 512 + 5 x 4096 + 28 x 4608 rows
    assert bench.gemm_in_rows_per_denoise(1, 512, 4096, 0, 16, True) == 16 * (5 * 512 + 5 * 4096 + 28 * 4608)
    # base CFG: text stage 1 (2 x 560 rows) once, image stage 1 every step, joint 2 x 16944 every step
    assert bench.gemm_in_rows_per_denoise(2, 560, 16384, 0, 50, False) == (
        5 * 2 * 560 + 50 * 5 * 16384 + 50 * 28 * 2 * 16944)
