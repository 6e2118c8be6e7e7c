"""Host logic of bench.py that needs no GPU: workload selection (--block), the
sweep's configurations, the traffic record keyed by the attention source's hash,
and the reference arm's JSON line on a bounded sample."""

import argparse
import hashlib
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
    with open(bench.ATTN_SRC, "rb") as f:
        sha = hashlib.sha256(f.read()).hexdigest()
    for key, rec in bench.ATTN_TRAFFIC.items():
        got = bench._attn_traffic(key)
        if sha.startswith(rec["src"]):
            assert got == rec["bytes"]
        else:
            assert got is None
    assert bench._attn_traffic("no-such-workload") is None


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
