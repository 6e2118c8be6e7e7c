"""The two forms of 2^x in the attention softmax, held to their error bounds on the GPU
against fp64 (GSRS §A.1: the online softmax's exponentials; the base-2 form with the
scale folded in is this build's reading). The FMA-pipe form is a Cody-Waite reduction
with a cubic minimax polynomial; the MUFU form is ex2.approx."""

import numpy as np
import pytest
import torch

import block_sparse_attention_video_b200 as F

pytestmark = pytest.mark.gpu


def _run(x_np):
    dev = torch.device("cuda")
    x = torch.from_numpy(x_np.astype(np.float32)).to(dev)
    y_fma = torch.full_like(x, float("nan"))
    y_mufu = torch.full_like(x, float("nan"))
    F.fvattn_exp2_selftest(x, y_fma, y_mufu)
    torch.cuda.synchronize()
    return x.cpu().numpy().astype(np.float64), y_fma.cpu().numpy().astype(np.float64), \
        y_mufu.cpu().numpy().astype(np.float64)


def test_fma_form_relative_error_below_1e4_over_the_softmax_range():
    # every exponent the softmax forms lies in (-inf, 8] (lazy rescale threshold),
    # 12 with the E4M3 path's shift of 4; a dense grid plus values at integers and halves
    grid = np.linspace(-125.0, 12.0, (1 << 20) + 1)
    marks = np.arange(-125.0, 12.5, 0.5)
    x, y_fma, y_mufu = _run(np.concatenate([grid, marks, [0.0, -0.0, 1e-7, -1e-7]]))
    ref = np.exp2(x)
    rel = np.abs(y_fma / ref - 1.0)
    assert rel.max() < 1e-4, (rel.max(), x[rel.argmax()])
    # the MUFU form: the hardware approximation, far tighter
    ok = x >= -125.0
    rel_m = np.abs(y_mufu[ok] / ref[ok] - 1.0)
    assert rel_m.max() < 2e-6, (rel_m.max(), x[ok][rel_m.argmax()])


def test_fma_form_clamps_below_minus_125_and_odd_counts():
    # masked keys reach the exponentials as -inf: the FMA form gives 2^-125 there (the
    # MUFU form 0); an odd count exercises the last unpaired element
    x_in = np.array([-126.0, -200.0, -1e30, -np.inf, -125.0, 0.0, 3.0], dtype=np.float64)
    x, y_fma, y_mufu = _run(x_in)
    low = x < -125.0
    assert np.all(np.abs(y_fma[low] / 2.0 ** -125 - 1.0) < 1e-4), y_fma[low]
    assert y_mufu[np.isinf(x)][0] == 0.0
    assert abs(y_fma[-2] - 1.0) < 1e-4 and abs(y_fma[-1] / 8.0 - 1.0) < 1e-4


def test_empty_input_launches_nothing():
    dev = torch.device("cuda")
    e = torch.empty(0, dtype=torch.float32, device=dev)
    F.fvattn_exp2_selftest(e, e.clone(), e.clone())
