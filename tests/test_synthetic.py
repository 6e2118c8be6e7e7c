"""The seeded input generator: deterministic, shaped as the workloads state."""

import math

import torch

import synthetic as S


def test_workload_shapes():
    w = S.WORKLOADS["wan14b-720p"]
    assert (w.N, w.nb, w.H, w.d, w.block) == (75600, 591, 40, 128, 128)
    assert w.N - (w.nb - 1) * w.block == 80
    assert S.WORKLOADS["wan1.3b-480p"].N == 32760 and S.WORKLOADS["wan1.3b-480p"].nb == 256
    assert S.WORKLOADS["tiny"].nb == 4
    sweep = S.sweep_workloads()
    assert len(sweep) == 36 and {s.block for s in sweep} == {64, 128}


def test_make_qkv_deterministic_and_dtypes():
    w = S.WORKLOADS["tiny"]
    a = S.make_qkv(w)
    b = S.make_qkv(w)
    for x, y in zip(a, b):
        assert torch.equal(x, y) and x.dtype == torch.float32 and x.shape == (1, 2, 256, 64)
    # head 1 of q is the peaky head (scaled by 3)
    assert a[0][0, 1].std() > 2.5 * a[0][0, 0].std()
    v = S.Workload("t", 1, 3, 64, "bf16", (3, 8, 8), (1, 8, 8), 64, 0.9, 1, seed=4,
                   temp=("loguniform", 0.3, 6.0))
    q, k, vv = S.make_qkv(v)
    assert q.dtype == torch.bfloat16 and q.shape == (1, 3, 192, 64)


def test_positional_code_unit_rms_and_smooth():
    pe = S.positional_code((6, 10, 12), 128)
    rms = pe.pow(2).mean().sqrt().item()
    assert abs(rms - 1.0) < 0.1
    # neighbouring tokens are more similar than distant ones
    near = (pe[0] * pe[1]).sum().item()
    far = (pe[0] * pe[-1]).sum().item()
    assert near > far


def test_temperatures_in_range():
    for name in ("wan1.3b-480p", "wan14b-480p", "wan14b-720p"):
        w = S.WORKLOADS[name]
        t = S.temperatures(w)
        _, lo, hi = w.temp
        assert t.shape == (w.H,) and float(t.min()) >= lo - 1e-6 and float(t.max()) <= hi + 1e-6
        assert math.isfinite(float(t.sum()))
