"""Host logic of bench.py that needs no GPU: workload selection (--block), the
sweep's configurations, the traffic record keyed by the attention source's hash,
and the reference arm's JSON line on a bounded sample."""

import argparse
import json

import pytest

import bench
import synthetic as S


def _args(**kw):
    base = dict(workload="wan14b-720p", block=None)
    base.update(kw)
    return argparse.Namespace(**base)


def test_block_option_switches_tiles_and_name():
    w = bench._workload(_args(block=64))
    assert (w.block, w.tile, w.name) == (64, (1, 8, 8), "wan14b-720p-bs64")
    assert w.grid == S.WORKLOADS["wan14b-720p"].grid and w.H == 40
    assert bench._workload(_args(block=128)) == S.WORKLOADS["wan14b-720p"]
    assert bench._workload(_args()) == S.WORKLOADS["wan14b-720p"]
    w480 = bench._workload(_args(workload="wan14b-480p", block=64))
    assert (w480.block, w480.tile, w480.N) == (64, (1, 8, 8), 32760)


def test_sweep_covers_p_kmin_and_block_sizes():
    ws = S.sweep_workloads()
    assert len(ws) == 36
    assert {w.p for w in ws} == {0.5, 0.7, 0.9, 0.95, 0.99, 1.0}
    assert {w.k_min for w in ws} == {1, 4, 16}
    assert {(w.block, w.tile) for w in ws} == {(128, (2, 8, 8)), (64, (1, 8, 8))}
    assert len({w.name for w in ws}) == 36


def test_traffic_is_reported_only_for_the_captured_source():
    with open(bench.ATTN_SRC) as f:
        sha = bench._code_hash(f.read())
    for kind, rec in bench.ATTN_TRAFFIC.items():
        got, note = bench._attn_traffic(kind, 2.0e9)
        if rec["bytes_480p"] is not None and sha.startswith(rec["src"]):
            assert got == pytest.approx(rec["bytes_480p"] / rec["algorithmic_480p"] * 2.0e9)
            assert "480p" in note
        else:
            assert got is None and note
    assert bench._attn_traffic("no-such-kind", 1.0) == (None, "no capture recorded")


def test_reference_arm_line(capsys):
    rc = bench.main(["--impl", "reference", "--workload", "wan1.3b-480p", "--block", "64", "--steps", "1",
                     "--warmup", "3", "--cpu-budget", "2"])
    assert rc == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["config"]["workload"] == "wan1.3b-480p-bs64" and line["config"]["block"] == 64
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["value"] > 0


def test_reference_arm_config_matches_the_gpu_arm(capsys):
    rc = bench.main(["--impl", "reference", "--workload", "tiny", "--steps", "1", "--warmup", "3"])
    assert rc == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["config"] == bench.bench_config(S.WORKLOADS["tiny"], 1)


def test_hbm_bytes_of_the_720p_call():
    w = S.WORKLOADS["wan14b-720p"]
    nb = w.nb
    hb = bench.hbm_bytes(w, nb, cnt_sum=1000)
    R = 40 * 75600 * 128 * 2
    P = 40 * nb * 128 * 128 * 2
    assert hb["permute_v"] == R + P and hb["inverse"] == 2 * R
    assert hb["route"] == 2 * R + 2 * P + 2 * 40 * nb * 128 * 4 + 4 * 1000 + 4 * 40 * nb
    total = sum(hb.values()) / 1e9
    assert 6.1 < total < 6.3


def test_oracle_check_on_the_oracles_own_result():
    """Lists and outputs taken from the oracle itself: no mismatch, zero error."""
    import math

    import numpy as np

    import oracle as O
    w = S.WORKLOADS["tiny"]
    q, k, v = (x.numpy() for x in S.make_qkv(w, device="cpu"))
    orc = O.route(q, k, w.grid6, w.block, w.p, w.k_min)
    nb = w.nb
    idx = np.zeros((w.B, w.H, nb, nb), dtype=np.int32)
    for r in np.ndindex(*orc["cnt"].shape):
        c = int(orc["cnt"][r])
        idx[r][:c] = np.sort(orc["order"][r][:c])
    cnt = orc["cnt"].astype(np.int32)
    mask = O.selection_mask(orc["order"], orc["cnt"])
    perm = orc["perm"]
    op = O.masked_attention(*(O.permute(x, perm, w.block) for x in (q, k, v)), mask, w.N, w.block,
                            1.0 / math.sqrt(w.d))
    mp, err, route_s, attn_s, flops, blocks = bench.oracle_check(
        w, q, k, v, idx, cnt, op, range(w.H), per_head=2, rng=np.random.default_rng(0))
    assert mp["mismatched"] == 0 and mp["hard"] == 0 and mp["heads"] == w.H
    assert mp["rows"] == w.H * nb and mp["selected_pairs"] == int(cnt.sum())
    assert err["max_abs"] < 1e-12 and err["within_tolerance"] and blocks >= w.H
    assert flops > 0 and route_s >= 0 and attn_s >= 0
    # a planted wrong output row is seen
    op[0, 0, 0, 0] += 1.0
    rng = np.random.default_rng(0)
    _, err2, *_ = bench.oracle_check(w, q, k, v, idx, cnt, op, [0], per_head=nb, rng=rng)
    assert err2["max_abs"] >= 0.999 and not err2["within_tolerance"]


def test_code_hash_ignores_comments_only():
    code = "int f(int x) {\n  return x + 1;  // add one\n}\n"
    assert bench._code_hash(code) == bench._code_hash("/* doc */\nint f(int x) {\n  return x + 1;\n}\n")
    assert bench._code_hash(code) != bench._code_hash(code.replace("+ 1", "+ 2"))
