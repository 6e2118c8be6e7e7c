"""Benchmark of the block-sparse attention path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl fvattn|reference]
                    [--workload wan14b-720p] [--no-e2e] [--no-cpu-baseline]

One step = one attention call of the whole path over one synthetic input
already resident in HBM: route (tile permutation of Q and K fused with
block-mean pooling, block scores, Top-p + Top-k floor, lists, per-head work),
permutation of V, block-sparse attention, inverse permutation of the output.
Throughput = effective TFLOP/s counted over the selected blocks only
(4 * d * sum over selected (query block, key block) pairs of
valid_query_rows * valid_keys), per step and per attention launch. The
build's own dense kernel is timed beside it at the same shape.

Multi-GPU (torchrun): every rank runs its own independent call (weak
scaling, no collective on the data path); the timed region is bracketed by
barriers and the max over ranks is reported.

--impl reference times the fp64 oracle (the CPU reference of this method) on
the host cores on a bounded sample of the same workload.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synthetic as S  # noqa: E402

METRIC = "sparse attn ms/call & effective TFLOP/s (Wan-14B 720p shape) vs own dense"


# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one attention
# launch from a one-pass ncu capture on the Wan-14B 480p shape (the size a
# capture may hold), with the algorithmic bytes of that launch (Q, K, V read
# once, O written once) and the prefix of _code_hash of the kernel source it was
# taken on (comments do not count). A 720p launch's traffic is reported as the
# 480p traffic scaled by the ratio of algorithmic bytes: the working set of the
# work units in flight (about one head's K and V) fits in L2 at both sizes, so the
# re-read factor carries over. After any change of the code the traffic is unknown
# and reported as null.
ATTN_TRAFFIC = {
    # 1,022,893,568 read + 320,081,408 written; Q, K, V, O at 2 B x 40 x 256 x 128 x 128
    "bf16": {"bytes_480p": 1022893568 + 320081408, "algorithmic_480p": 4 * 40 * 256 * 128 * 128 * 2,
             "src": "729c0bf9fa452b22"},
    # 846,904,576 read + 315,604,736 written; Q, K, O at 2 B and the E4M3 V at 1 B
    "fp8v": {"bytes_480p": 846904576 + 315604736, "algorithmic_480p": 7 * 40 * 256 * 128 * 128,
             "src": "729c0bf9fa452b22"},
}
ATTN_SRC = os.path.join(ROOT, "block_sparse_attention_video_b200", "csrc", "attn_sm100.cu")


# A 128 x 256 x 16 bf16 tcgen05.mma (kind::f16, fp32 accumulate) takes 128 SM cycles:
# 8,192 FLOP per clock per SM on the tensor pipe.
TENSOR_BF16_FLOP_PER_CLK_SM = 8192


def _frac_at_clock(achieved_tflops: float, clocks, dev):
    if not clocks or not clocks.get("sm_mhz"):
        return None
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    peak = TENSOR_BF16_FLOP_PER_CLK_SM * sms * clocks["sm_mhz"] * 1e6 / 1e12
    return achieved_tflops / peak


def _code_hash(text: str) -> str:
    """sha256 of a C++/CUDA source with its comments and blank lines removed, so that an
    edit of comments alone keeps a recorded measurement of the code valid."""
    import hashlib
    import re
    t = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    t = re.sub(r"//[^\n]*", "", t)
    lines = [ln.rstrip() for ln in t.splitlines() if ln.strip()]
    return hashlib.sha256("\n".join(lines).encode()).hexdigest()


def _attn_traffic(kind: str, algorithmic_bytes: float):
    """(scaled DRAM bytes per launch, note) for the current kernel source, or (None, why)."""
    import hashlib
    rec = ATTN_TRAFFIC.get(kind)
    if rec is None or rec["bytes_480p"] is None:
        return None, "no capture recorded"
    try:
        with open(ATTN_SRC) as f:
            sha = _code_hash(f.read())
    except OSError:
        return None, "kernel source not found"
    if not sha.startswith(rec["src"]):
        return None, "kernel code changed since the capture"
    ratio = rec["bytes_480p"] / rec["algorithmic_480p"]
    return ratio * algorithmic_bytes, (f"ncu one-pass DRAM bytes at the Wan-14B 480p shape "
                                       f"({rec['bytes_480p'] / 1e9:.3f} GB, {ratio:.3f}x its algorithmic bytes), "
                                       f"scaled to this launch's algorithmic bytes")


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            pk = json.load(f)
        return dict(hbm=float(pk["hbm_gbs"]), bf16=float(pk["bf16_tflops"]),
                    bf16_sus=float(pk["bf16_tflops_sustained"]), source="measured")
    except (OSError, KeyError, ValueError):
        return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, source="fallback")


def effective_flops(kv_idx: np.ndarray, kv_cnt: np.ndarray, N: int, bs: int, d: int) -> float:
    """4*d*sum over selected (i, j) of valid_rows(i) * valid_keys(j)."""
    nb = kv_cnt.shape[-1]
    n = np.full(nb, bs, dtype=np.float64)
    n[-1] = N - (nb - 1) * bs
    valid = np.arange(kv_idx.shape[-1]) < kv_cnt[..., None]
    keys = np.where(valid, n[np.clip(kv_idx, 0, nb - 1)], 0.0).sum(-1)      # [B,H,nb]
    return float(4.0 * d * (keys * n[None, None, :]).sum())


def dense_flops(B, H, N, d) -> float:
    return 4.0 * B * H * float(N) * float(N) * d


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms during a region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"fvattn_clocks_{os.getpid()}.csv")

    def __enter__(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=self.fh, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.fh.close()

    def summary(self):
        if self.proc is None:
            return None
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append((float(parts[1]), float(parts[2]), parts[5:9], float(parts[3])))
                except ValueError:
                    continue
        try:
            os.remove(self.path)
        except OSError:
            pass
        if not rows:
            return None
        load = [r for r in rows if r[3] > 200.0] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in load for i, v in enumerate(r[2]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in load), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows), "samples_under_load": len(load),
                "power_w_max": max(r[3] for r in rows)}


def _dist_setup(n_gpus, backend="nccl"):
    """One process per GPU (torchrun env). The data path has no collective: the
    group only carries the barriers and the max over ranks of the timings.
    backend "gloo" (CPU tests) leaves the CUDA device alone."""
    import datetime
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    timeout = datetime.timedelta(seconds=120)
    if world > 1:
        import torch.distributed as dist
        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", device_id=torch.device("cuda", local), timeout=timeout)
        else:
            dist.init_process_group(backend, timeout=timeout)
        return dist, rank, world, local
    if backend == "nccl":
        torch.cuda.set_device(local)
    return None, 0, 1, local


def _barrier(dist):
    if dist is not None:
        dist.barrier()


def _max_over_ranks(dist, v: float, device="cuda") -> float:
    if dist is None:
        return v
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def hbm_bytes(w, nb: int, cnt_sum: int) -> dict:
    """Algorithmic HBM bytes of the bandwidth-bound kernels of one call.

    route:   Q and K read in raster order (2 R), written in tile order with pad
             rows (2 P), the fp32 block means (2 x nb x d x 4 per head) and the
             selected list entries with their counts (4 B each);
    permute: V read (R) and written in tile order (P);
    inverse: the N valid output rows read and written back in raster order (2 R).
    R = B*H*N*d*2 bytes, P = B*H*Npad*d*2 bytes (bf16)."""
    bh = w.B * w.H
    R = bh * w.N * w.d * 2
    P = bh * nb * w.block * w.d * 2
    route = 2 * R + 2 * P + 2 * bh * nb * w.d * 4 + 4 * cnt_sum + 4 * bh * nb
    return {"route": route, "permute_v": R + P, "inverse": 2 * R}


def _sample_query_blocks(rng, nb, cnt_row_max, per_head):
    picks = set(rng.permutation(nb)[:per_head].tolist())
    picks.add(nb - 1)                      # the ragged tail block
    picks.add(int(cnt_row_max))            # the head's heaviest row
    return sorted(picks)


def oracle_check(w, qn, kn, vn, idx, cnt, op_perm, heads, per_head, rng, budget_s=None):
    """The fp64 oracle on the host cores against one GPU call (test infrastructure:
    runs only in the cpu_baseline leg and the sweep's parity check).

    Routing of the given heads (permute, pool, scores, Top-p + floor) gives the
    mask parity of the GPU's lists; masked attention of sampled query blocks of
    those heads on the GPU's own mask gives the GPU output's error on those rows
    (op_perm: the GPU output in tile order [B,H,Npad,d]). Returns (parity dict,
    error dict, route seconds, attention seconds, attention FLOPs)."""
    import oracle as O
    from oracle.mask_parity import compare_masks, mask_from_lists, summary
    nb = w.nb
    heads = list(heads)
    t0 = time.perf_counter()
    orc = O.route(qn[:, heads], kn[:, heads], w.grid6, w.block, w.p, w.k_min)
    route_s = time.perf_counter() - t0
    mask = mask_from_lists(idx[:, heads], cnt[:, heads], nb)
    mp = summary(compare_masks(mask, orc, w.p))
    mp["heads"] = len(heads)
    perm = orc["perm"]
    n = np.full(nb, w.block, dtype=np.float64)
    n[-1] = w.N - (nb - 1) * w.block
    scale = 1.0 / math.sqrt(w.d)
    flops, blocks, emax, esum, ecount = 0.0, 0, 0.0, 0.0, 0
    t1 = time.perf_counter()
    for hi, h in enumerate(heads):
        qh, kh, vh = (O.permute(x[0, h].astype(np.float64), perm, w.block) for x in (qn, kn, vn))
        for i in _sample_query_blocks(rng, nb, np.argmax(cnt[0, h]), per_head):
            ref = O.masked_attention_rows(qh, kh, vh, mask[0, hi, i], w.N, w.block, scale, int(i))
            got = op_perm[0, h, i * w.block:i * w.block + ref.shape[0]].astype(np.float64)
            e = np.abs(got - ref)
            emax = max(emax, float(e.max()))
            esum += float(e.sum())
            ecount += e.size
            flops += 4.0 * w.d * n[i] * n[mask[0, hi, i]].sum()
            blocks += 1
        if budget_s is not None and time.perf_counter() - t1 > budget_s:
            break
    attn_s = time.perf_counter() - t1
    mean = esum / max(1, ecount)
    err = {"query_blocks": blocks, "max_abs": emax, "mean_abs": mean,
           "tolerance": {"max_abs": 2e-2, "mean_abs": 2e-3},
           "within_tolerance": bool(emax <= 2e-2 and mean <= 2e-3),
           "against": "fp64 oracle masked attention on the GPU's own mask"}
    return mp, err, route_s, attn_s, flops, blocks


LVSA_WINDOW, LVSA_PERIOD, LVSA_STEP = 2, 8, 0
GSRS_SEARCH_P = 0.9
E2E_HEAD_GROUPS = 10


def _median_ms(fn, stream, warmup, reps):
    for _ in range(max(1, warmup)):
        fn()
    ts = []
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b))
    return statistics.median(ts)


def run_lvsa(F, w, path, stream, warmup, eff_flops_fn):
    """The LVSA static mask (window + rotating global frames) on the same tensors."""
    dev = path.qp.device
    idx = torch.empty_like(path.kv_idx)
    cnt = torch.empty_like(path.kv_cnt)
    hw = torch.empty_like(path.head_work)
    ws = F.alloc_workspace(F.fvattn_workspace_bytes(F.FVATTN_OP_LVSA, w.B, w.H, w.N, w.d, w.block), dev)
    gen_ms = _median_ms(lambda: F.fvattn_lvsa_lists(path.grid, LVSA_WINDOW, LVSA_PERIOD, LVSA_STEP, idx, cnt,
                                                    hw, ws), stream, warmup, 3)
    attn_ms = _median_ms(lambda: F.fvattn_sparse_fwd(path.qp, path.kp, path.vp, path.op, idx, cnt, w.N,
                                                     w.block, path.ws_attn), stream, warmup, 3)
    if F.fvattn_workspace_status(ws) != F.FVATTN_OK or F.fvattn_workspace_status(path.ws_attn) != F.FVATTN_OK:
        raise RuntimeError("kernel status word set in the LVSA run")
    idx_np, cnt_np = idx.cpu().numpy(), cnt.cpu().numpy()
    eff = eff_flops_fn(idx_np, cnt_np, w.N, w.block, w.d)
    hwn = hw.cpu().numpy().astype(np.float64)
    return {"window": LVSA_WINDOW, "period": LVSA_PERIOD, "step": LVSA_STEP,
            "density": float(cnt_np.mean() / path.nb), "lists_ms": gen_ms, "attention_ms": attn_ms,
            "effective_tflops": eff / (attn_ms * 1e-3) / 1e12,
            "head_work_max_over_mean": float(hwn.max() / hwn.mean()), "_lists": (idx, cnt)}


def run_fp8v(F, w, path, stream, warmup, eff, q, k, v):
    """Attention with the per-channel E4M3 V (8-bit P.V product) on the routed lists
    of the timed call: the quantization step (alone, and fused with the permutation),
    the sparse and dense launches, the output's distance from the bf16-V launch on the
    same inputs, and the whole step with the E4M3 V (route, fused permutation and
    quantization of V, attention, inverse permutation)."""
    dev = path.qp.device
    vq = torch.empty(path.vp.shape, dtype=torch.uint8, device=dev)
    vs = torch.empty((w.B, w.H, w.d), dtype=torch.float32, device=dev)
    wsq = F.alloc_workspace(F.fvattn_workspace_bytes(F.FVATTN_OP_QUANT_V, w.B, w.H, w.N, w.d, w.block), dev)
    quant_ms = _median_ms(lambda: F.fvattn_quantize_v(path.vp, vq, vs, w.N, w.block, wsq), stream, warmup, 5)
    out8 = torch.empty_like(path.op)
    sparse_ms = _median_ms(lambda: F.fvattn_sparse_fwd_fp8v(path.qp, path.kp, vq, vs, out8, path.kv_idx,
                                                            path.kv_cnt, w.N, w.block, path.ws_attn),
                           stream, warmup, 3)
    F.fvattn_sparse_fwd(path.qp, path.kp, path.vp, path.op, path.kv_idx, path.kv_cnt, w.N, w.block,
                        path.ws_attn)
    diff = (out8[:, :, :w.N].float() - path.op[:, :, :w.N].float()).abs()
    dense_ms = _median_ms(lambda: F.fvattn_dense_fwd_fp8v(path.qp, path.kp, vq, vs, out8, w.N, w.block,
                                                          path.ws_attn), stream, warmup, 3)
    fused_ms = _median_ms(lambda: F.fvattn_permute_quantize_v(v, path.grid, vq, vs, wsq), stream, warmup, 5)
    p8 = F.FVAttnPath(w.B, w.H, w.grid, w.tile, w.block, w.d, torch.bfloat16, w.p, w.k_min, device=dev,
                      v_format="e4m3")

    def step8():
        p8.route(q, k)
        p8.prepare_v(v)
        p8.attend()
        F.fvattn_permute(p8.op, p8.out, p8.grid, inverse=True)

    step_ms = _median_ms(step8, stream, warmup, 5)
    same_codes = bool(torch.equal(p8.vq, vq) and torch.equal(p8.vscale, vs))
    if F.fvattn_workspace_status(wsq) != F.FVATTN_OK or F.fvattn_workspace_status(path.ws_attn) != F.FVATTN_OK \
            or F.fvattn_workspace_status(p8.ws_attn) != F.FVATTN_OK or F.fvattn_workspace_status(p8.ws_quant) != F.FVATTN_OK:
        raise RuntimeError("kernel status word set in the FP8 V run")
    del p8
    torch.cuda.empty_cache()
    v_bytes = w.B * w.H * w.N * w.d * 2
    q_bytes = w.B * w.H * path.npad * w.d
    d_flops = dense_flops(w.B, w.H, w.N, w.d)
    return {"format": "E4M3, one fp32 scale per (b, h, channel); P rounded to E4M3 in the kernel",
            "quantize_ms": quant_ms,
            "quantize_gbs": (v_bytes + q_bytes) / (quant_ms * 1e-3) / 1e9,
            "quantize_bytes": {"algorithmic": v_bytes + q_bytes, "moved": 2 * v_bytes + q_bytes,
                               "note": "two passes over V: channel maxima, then encoding"},
            "permute_quantize_ms": fused_ms,
            "permute_quantize_gbs": (2 * v_bytes + q_bytes) / (fused_ms * 1e-3) / 1e9,
            "permute_quantize_note": "fvattn_permute_quantize_v from the raster-order V: reads V twice "
                                     "(maxima, gather + encode), writes the codes; equal codes to permute + "
                                     f"quantize: {same_codes}",
            "step_ms": step_ms,
            "step_note": "route + fused permutation/quantization of V + sparse attention (E4M3 P.V) + inverse",
            "attention_ms": sparse_ms, "effective_tflops": eff / (sparse_ms * 1e-3) / 1e12,
            "dense_attention_ms": dense_ms, "dense_tflops": d_flops / (dense_ms * 1e-3) / 1e12,
            "max_abs_diff_vs_bf16_v": float(diff.max()), "mean_abs_diff_vs_bf16_v": float(diff.mean())}


def run_hilbert(F, w, q, k, v, stream, warmup, eff_flops_fn):
    """The same call with blocks in Hilbert-curve order instead of 3-D tiles."""
    dev = q.device
    hpath = F.FVAttnPath(w.B, w.H, w.grid, w.tile, w.block, w.d, torch.bfloat16, w.p, w.k_min, device=dev,
                         order="hilbert")
    # the table build alone (once per grid), its buffers already cached by the first build
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    F.fvattn_hilbert_table(w.grid, w.block, dev)
    t1.record(stream)
    torch.cuda.synchronize()
    table_ms = t0.elapsed_time(t1)
    hpath.route(q, k)
    F.fvattn_permute(v, hpath.vp, hpath.grid)
    attn_ms = _median_ms(lambda: hpath.attend(), stream, warmup, 3)
    route_ms = _median_ms(lambda: hpath.route(q, k), stream, warmup, 3)
    if F.fvattn_workspace_status(hpath.ws_route) != F.FVATTN_OK or \
            F.fvattn_workspace_status(hpath.ws_attn) != F.FVATTN_OK:
        raise RuntimeError("kernel status word set in the Hilbert-order run")
    idx_np, cnt_np = hpath.kv_idx.cpu().numpy(), hpath.kv_cnt.cpu().numpy()
    eff = eff_flops_fn(idx_np, cnt_np, w.N, w.block, w.d)
    hwn = hpath.head_work.cpu().numpy().astype(np.float64)
    diag = run_diag(F, w, hpath, stream, warmup)
    out = {"table_build_ms": table_ms, "route_ms": route_ms, "density": float(cnt_np.mean() / hpath.nb),
           "attention_ms": attn_ms, "effective_tflops": eff / (attn_ms * 1e-3) / 1e12,
           "head_work_max_over_mean": float(hwn.max() / hwn.mean()),
           "recall_of_routed_mask": diag["recall_of_routed_mask"]}
    del hpath
    torch.cuda.empty_cache()
    return out


def run_diag(F, w, path, stream, warmup, lvsa_lists=None):
    dev = path.qp.device
    nb, npad = path.nb, path.npad
    lse = torch.empty((w.B, w.H, npad), dtype=torch.float32, device=dev)
    blse = torch.empty((w.B, w.H, nb, npad), dtype=torch.float32, device=dev)
    imp = torch.empty((w.B, w.H, nb, nb), dtype=torch.float32, device=dev)
    rec = torch.empty((w.B, w.H, nb), dtype=torch.float32, device=dev)
    wsd = F.alloc_workspace(F.fvattn_workspace_bytes(F.FVATTN_OP_DIAG, w.B, w.H, w.N, w.d, w.block), dev)

    def timed(fn, reps):
        for _ in range(max(1, warmup)):
            fn()
        ts = []
        for _ in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        return statistics.median(ts)

    sparse_ms = timed(lambda: F.fvattn_sparse_fwd(path.qp, path.kp, path.vp, path.op, path.kv_idx,
                                                  path.kv_cnt, w.N, w.block, path.ws_attn), 3)
    sparse_blse_ms = timed(lambda: F.fvattn_sparse_fwd(path.qp, path.kp, path.vp, path.op, path.kv_idx,
                                                       path.kv_cnt, w.N, w.block, path.ws_attn,
                                                       lse=lse, block_lse=blse), 3)
    imp_ms = timed(lambda: F.fvattn_block_importance(blse, lse, imp, w.N, w.block, wsd,
                                                     kv_idx=path.kv_idx, kv_cnt=path.kv_cnt), 3)
    sparse_sum = float(imp.sum(-1).sub(1).abs().max())
    # GSRS search step: Top-p (with the Top-k floor) on the exact importance of the
    # routed candidates gives the next, smaller mask inside them.
    idx2 = torch.empty_like(path.kv_idx)
    cnt2 = torch.empty_like(path.kv_cnt)
    hw2 = torch.empty_like(path.head_work)
    select_ms = timed(lambda: F.fvattn_select_topp(imp, w.N, w.block, GSRS_SEARCH_P, w.k_min, idx2, cnt2, hw2,
                                                   wsd), 3)
    F.fvattn_dense_fwd(path.qp, path.kp, path.vp, path.op, w.N, w.block, path.ws_attn, lse=lse,
                       block_lse=blse)
    F.fvattn_block_importance(blse, lse, imp, w.N, w.block, wsd)
    F.fvattn_attention_recall(imp, path.kv_idx, path.kv_cnt, rec, w.N, w.block, wsd)
    rec2 = torch.empty_like(rec)
    F.fvattn_attention_recall(imp, idx2, cnt2, rec2, w.N, w.block, wsd)
    rec_lvsa = None
    if lvsa_lists is not None:
        rec_lvsa = torch.empty_like(rec)
        F.fvattn_attention_recall(imp, lvsa_lists[0], lvsa_lists[1], rec_lvsa, w.N, w.block, wsd)
    torch.cuda.synchronize()
    if F.fvattn_workspace_status(wsd) != F.FVATTN_OK or F.fvattn_workspace_status(path.ws_attn) != F.FVATTN_OK:
        raise RuntimeError("kernel status word set in the diagnostic")
    r = rec.float()
    out = {"sparse_attention_ms": sparse_ms, "sparse_attention_with_block_lse_ms": sparse_blse_ms,
           "block_lse_overhead": sparse_blse_ms / sparse_ms - 1.0, "importance_ms": imp_ms,
           "sparse_importance_row_sum_max_err": sparse_sum,
           "recall_of_routed_mask": {"mean": float(r.mean()), "p05": float(r.flatten().quantile(0.05)),
                                     "min": float(r.min())},
           "note": "GSRS block importance from block log-sum-exps; recall = dense importance captured by the "
                   "routed lists",
           "search": {"p": GSRS_SEARCH_P, "k_min": w.k_min, "select_ms": select_ms,
                      "density": float(cnt2.float().mean() / nb),
                      "recall": {"mean": float(rec2.mean()), "p05": float(rec2.flatten().quantile(0.05)),
                                 "min": float(rec2.min())},
                      "note": "Top-p on the exact importance of the routed candidates (fvattn_select_topp)"}}
    if rec_lvsa is not None:
        rl = rec_lvsa.float()
        out["recall_of_lvsa_mask"] = {"mean": float(rl.mean()), "p05": float(rl.flatten().quantile(0.05)),
                                      "min": float(rl.min())}
    del blse, imp, idx2
    torch.cuda.empty_cache()
    return out


def replica_workload(w, rank: int):
    """Each rank runs an independent call of the same shape on its own inputs."""
    return w.replace(seed=w.seed + 1000 * rank)


def _workload(args):
    """The named workload; --block 64 runs it with 64-token blocks (1x8x8 tiles, as in the sweep)."""
    w = S.WORKLOADS[args.workload]
    if args.block and args.block != w.block:
        w = w.replace(name=f"{w.name}-bs{args.block}", block=args.block,
                      tile=(1, 8, 8) if args.block == 64 else (2, 8, 8))
    return w


def run_fvattn(args):
    import block_sparse_attention_video_b200 as F
    dist, rank, world, local = _dist_setup(args.gpus)
    w = _workload(args)
    dev = torch.device("cuda", local)
    q, k, v = S.make_qkv(replica_workload(w, rank), device=dev)
    path = F.FVAttnPath(w.B, w.H, w.grid, w.tile, w.block, w.d, torch.bfloat16, w.p, w.k_min, device=dev)
    stream = torch.cuda.current_stream()

    def step(ev=None):
        # ev: five events around the four calls (route, V permute, attention, inverse)
        if ev is not None:
            ev[0].record(stream)
        path.route(q, k)
        if ev is not None:
            ev[1].record(stream)
        F.fvattn_permute(v, path.vp, path.grid)
        if ev is not None:
            ev[2].record(stream)
        path.attend()
        if ev is not None:
            ev[3].record(stream)
        F.fvattn_permute(path.op, path.out, path.grid, inverse=True)
        if ev is not None:
            ev[4].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if F.fvattn_workspace_status(path.ws_route) != F.FVATTN_OK or \
            F.fvattn_workspace_status(path.ws_attn) != F.FVATTN_OK:
        raise RuntimeError("kernel status word set during warm-up")
    idx_np, cnt_np = path.kv_idx.cpu().numpy(), path.kv_cnt.cpu().numpy()
    eff = effective_flops(idx_np, cnt_np, w.N, w.block, w.d)
    density = float(cnt_np.mean() / path.nb)
    hw = path.head_work.cpu().numpy().astype(np.float64)
    work_ratio = float(hw.max() / hw.mean())

    # ---- timed region: K full steps, events around each call of a step
    ev = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(5)) for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    gpu_index = int(os.environ.get("CUDA_VISIBLE_DEVICES", str(local)).split(",")[local]) \
        if os.environ.get("CUDA_VISIBLE_DEVICES") else local
    with ClockSampler(gpu_index) as clk:
        _barrier(dist)
        torch.cuda.synchronize()
        start.record(stream)
        for s in range(args.steps):
            step(ev[s])
        end.record(stream)
        torch.cuda.synchronize()
        _barrier(dist)
    clocks = clk.summary()
    ms_step = start.elapsed_time(end) / args.steps

    def call_ms(i):
        return sum(e[i].elapsed_time(e[i + 1]) for e in ev) / len(ev)

    ms_route, ms_vperm, ms_attn, ms_inv = (call_ms(i) for i in range(4))
    ms_step_max = _max_over_ranks(dist, ms_step)
    launches_per_step = 9   # gather_pool, block scores, select rows, permute V, plan x3, attention, inverse

    # ---- the build's own dense kernel at the same shape
    dense_ms = []
    for it in range(args.warmup + max(2, args.steps // 2)):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        path.attend(dense=True)
        b.record(stream)
        torch.cuda.synchronize()
        if it >= args.warmup:
            dense_ms.append(a.elapsed_time(b))
    ms_dense = sum(dense_ms) / len(dense_ms)
    d_flops = dense_flops(w.B, w.H, w.N, w.d)

    # ---- GSRS diagnostic (outside the timed region): cost of recording block
    # log-sum-exps in the sparse launch, the importance kernel, and the attention
    # recall of the routed mask under the dense attention's block importance.
    hilbert = None
    if not args.no_hilbert:
        hilbert = run_hilbert(F, w, q, k, v, stream, args.warmup, eff_flops_fn=effective_flops)
    lvsa = None
    if not args.no_lvsa:
        lvsa = run_lvsa(F, w, path, stream, args.warmup, eff_flops_fn=effective_flops)
    diag = None
    if not args.no_diag:
        diag = run_diag(F, w, path, stream, args.warmup,
                        lvsa_lists=(lvsa.pop("_lists") if lvsa is not None else None))
    fp8v = None
    if not args.no_fp8v:
        fp8v = run_fp8v(F, w, path, stream, args.warmup, eff, q, k, v)
        fp8v["speedup_vs_bf16_v"] = ms_attn / fp8v["attention_ms"]
        fp8v["step_speedup_vs_bf16_step"] = ms_step / fp8v["step_ms"]
        fp8v["dense_speedup_vs_bf16_v"] = ms_dense / fp8v["dense_attention_ms"]

    # ---- e2e through the public API with pinned host buffers: every step uploads its
    # q, k, v and downloads its output; HostPipeline overlaps the copies of
    # neighbouring steps with the kernels of the current one.
    e2e = None
    if not args.no_e2e:
        hq, hk, hv = (x.cpu().pin_memory() for x in (q, k, v))
        hout = torch.empty(path.out.shape, dtype=path.out.dtype).pin_memory()
        groups = E2E_HEAD_GROUPS if (w.B == 1 and w.H >= 2 * E2E_HEAD_GROUPS) else 1
        pipe = F.HostPipeline(path, head_groups=groups)
        pipe.run([(hq, hk, hv)] * max(1, args.warmup), [hout] * max(1, args.warmup))
        torch.cuda.synchronize()
        e_steps = max(2, args.steps)
        a = torch.cuda.Event(enable_timing=True)
        _barrier(dist)
        a.record(stream)
        end_ev = pipe.run([(hq, hk, hv)] * e_steps, [hout] * e_steps, start_event=a)
        b = torch.cuda.Event(enable_timing=True)
        b.record(stream)
        torch.cuda.synchronize()
        _barrier(dist)
        ms_e2e = _max_over_ranks(dist, a.elapsed_time(b) / e_steps)
        if F.fvattn_workspace_status(path.ws_attn) != F.FVATTN_OK:
            raise RuntimeError("kernel status word set in the e2e run")
        in_bytes = sum(x.numel() * x.element_size() for x in (hq, hk, hv))
        e2e = {"value": world * eff / (ms_e2e * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": ms_e2e,
               "h2d_bytes_per_step": int(in_bytes), "d2h_bytes_per_step": int(hout.numel() * hout.element_size()),
               "steps": e_steps, "head_groups": groups,
               "overlap": "copies of neighbouring steps overlap the current step's kernels; each step runs as "
                          f"{groups} head range(s) on separate streams, so compute starts after the first "
                          "range's upload and outputs go down range by range"}
        del pipe
        torch.cuda.empty_cache()

    if rank != 0:
        if dist is not None:
            dist.destroy_process_group()
        return 0

    pk = _peaks()
    achieved = eff / (ms_attn * 1e-3) / 1e12
    hb = hbm_bytes(w, path.nb, int(cnt_np.astype(np.int64).sum()))
    attn_alg_bytes = 4 * w.B * w.H * path.nb * w.block * w.d * 2
    traffic_bf16, traffic_bf16_note = _attn_traffic("bf16", attn_alg_bytes)
    hbm_ms = ms_route + ms_vperm + ms_inv
    hbm_achieved = (hb["route"] + hb["permute_v"] + hb["inverse"]) / (hbm_ms * 1e-3) / 1e9
    line = {
        "metric": METRIC,
        "value": world * eff / (ms_step_max * 1e-3) / 1e12,
        "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_step_max,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": bench_config(w, world),
        "ms_per_call": ms_step_max,
        "ms_per_call_by_step": {"route": ms_route, "permute_v": ms_vperm, "attention": ms_attn,
                                "inverse_permute": ms_inv},
        "attention_ms_per_launch": ms_attn,
        "effective_tflop_per_call": eff / 1e12,
        "density": density,
        "head_work_max_over_mean": work_ratio,
        "dense": {"attention_ms_per_launch": ms_dense, "tflops": d_flops / (ms_dense * 1e-3) / 1e12,
                  "tflop_per_call": d_flops / 1e12},
        "speedup_vs_dense_attention": ms_dense / ms_attn,
        "roofline": {"bound": "tensor", "kernel": "attn_fwd_sm100_kernel", "achieved": achieved,
                     "peak": pk["bf16_sus"], "unit": "TFLOP/s", "frac": achieved / pk["bf16_sus"],
                     "peak_kind": f"{pk['source']} bf16 sustained (kernel timed inside a long step)",
                     "frac_of_burst_peak": achieved / pk["bf16"],
                     "frac_at_clock": _frac_at_clock(achieved, clocks, dev),
                     "frac_at_clock_note": "achieved / (8,192 bf16 FLOP per clock per SM x SMs x the median SM "
                                           "clock sampled in the timed region): the kernel's share of what the "
                                           "tensor pipes deliver at the clock it actually ran at",
                     "traffic": traffic_bf16, "traffic_note": traffic_bf16_note,
                     "traffic_unit": "bytes per launch (DRAM read + write)",
                     "algorithmic_bytes": attn_alg_bytes},
        "roofline_hbm": {"bound": "hbm", "kernels": "route (gather + pool, block scores, select) + V permute + "
                                                    "inverse permute",
                         "achieved": hbm_achieved, "peak": pk["hbm"], "unit": "GB/s",
                         "frac": hbm_achieved / pk["hbm"], "peak_kind": f"{pk['source']} HBM copy bandwidth",
                         "ms": hbm_ms, "algorithmic_bytes": hb,
                         "traffic": None,
                         "note": "CUDA events around each call inside the timed steps; bytes as in hbm_bytes()"},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
    }
    if e2e is not None:
        line["e2e"] = e2e
    if lvsa is not None:
        lvsa.pop("_lists", None)
        line["lvsa"] = lvsa
    if hilbert is not None:
        line["hilbert"] = hilbert
    if diag is not None:
        line["diag"] = diag
    if fp8v is not None:
        # Q.K^T stays bf16 and P.V runs on E4M3 at the nominal 2x rate: at equal halves of
        # the FLOPs the tensor-core ceiling is 4/3 of the bf16 one.
        a8 = eff / (fp8v["attention_ms"] * 1e-3) / 1e12
        p8 = pk["bf16_sus"] * 4.0 / 3.0
        fp8v["roofline"] = {"bound": "tensor", "kernel": "attn_fwd_sm100_kernel (E4M3 P.V)", "achieved": a8,
                            "peak": p8, "unit": "TFLOP/s", "frac": a8 / p8,
                            "traffic": _attn_traffic("fp8v", 7 * w.B * w.H * path.nb * w.block * w.d)[0],
                            # Q, K read (2 B each), E4M3 V read (1 B), O written (2 B) per element
                            "algorithmic_bytes": 7 * w.B * w.H * path.nb * w.block * w.d,
                            "peak_kind": f"{pk['source']} bf16 sustained x 4/3 (half the FLOPs at the "
                                         f"nominal fp8/bf16 ratio of 2)"}
        line["fp8v"] = fp8v
    if not args.no_cpu_baseline:
        # The timed call once more (the diagnostics above overwrite the output
        # buffer), then the oracle on the host cores: routing of every head for the
        # mask parity, masked attention of sampled query blocks for the output error
        # and the oracle's throughput.
        step()
        torch.cuda.synchronize()
        idx2, cnt2 = path.kv_idx.cpu().numpy(), path.kv_cnt.cpu().numpy()
        same_lists = bool(np.array_equal(cnt2, cnt_np) and all(
            np.array_equal(idx2[r][:c], idx_np[r][:c]) for r, c in np.ndenumerate(cnt_np)))
        cores = len(os.sched_getaffinity(0))
        qn, kn, vn = (x.float().cpu().numpy() for x in (q, k, v))
        op_perm = path.op.float().cpu().numpy()
        rng = np.random.default_rng(0)
        mp, err, route_s, attn_s, oflops, nblk = oracle_check(
            w, qn, kn, vn, idx2, cnt2, op_perm, range(w.H), per_head=2, rng=rng, budget_s=args.cpu_budget)
        mp["lists_identical_across_calls"] = same_lists
        del qn, kn, vn, op_perm
        tf = oflops / attn_s / 1e12
        line["mask_parity"] = mp
        line["output_error"] = err
        line["cpu_baseline"] = {
            "value": tf, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": f"fp64 oracle block-sparse attention of {nblk} query blocks of this call (the tail "
                      f"block, each head's heaviest row and random ones) on the GPU's mask, {attn_s:.1f} s; "
                      f"routing of all {w.H} heads {route_s:.1f} s",
            "oracle_ms_per_query_block": attn_s * 1e3 / max(1, nblk),
            "oracle_route_ms": route_s * 1e3,
            "extrapolated_call_ms": route_s * 1e3 + eff / (tf * 1e12) * 1e3,
            "extrapolated_note": "EXTRAPOLATED: measured routing of every head plus this call's effective "
                                 "FLOPs at the sampled blocks' oracle throughput"}
    print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()
    return 0


def bench_config(w, world: int) -> dict:
    """The config dict of the JSON line (the same for both arms)."""
    return {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "grid": list(w.grid),
            "tiles": list(w.tile), "block": w.block, "p": w.p, "k_min": w.k_min,
            "l2": f"inputs larger than L2 (Q, K, V {w.B * w.H * w.N * w.d * 2 / 1e6:.0f} MB each); no flush",
            "parallelism": f"independent replicas x{world}"}


def run_reference(args):
    """The oracle timed on the host cores on a bounded sample of the workload."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle as O
    w = _workload(args)
    cores = len(os.sched_getaffinity(0))
    q, k, v = S.make_qkv(w, device="cpu")
    perm = O.tile_order(*w.grid6)
    scale = 1.0 / math.sqrt(w.d)
    nb = w.nb
    n = np.full(nb, w.block, dtype=np.float64)
    n[-1] = w.N - (nb - 1) * w.block
    rng = np.random.default_rng(0)

    def one_step(h):
        # one head: route (permute, pool, scores, Top-p) + attention of 2 query blocks
        qh, kh, vh = (O.permute(x[0, h].float().numpy().astype(np.float64), perm, w.block) for x in (q, k, v))
        qbar, kbar = O.block_mean_pool(qh, w.N, w.block), O.block_mean_pool(kh, w.N, w.block)
        s = O.block_scores(qbar, kbar, scale)
        flops = 0.0
        for i in rng.permutation(nb)[:2]:
            order, c = O.topp_topk_select(s[i], w.p, w.k_min)
            mrow = np.zeros(nb, dtype=bool)
            mrow[order[:c]] = True
            O.masked_attention_rows(qh, kh, vh, mrow, w.N, w.block, scale, int(i))
            flops += 4.0 * w.d * n[i] * n[mrow].sum()
        return flops

    for h in range(args.warmup):
        one_step(h % w.H)
    t0 = time.perf_counter()
    flops = 0.0
    for s_ in range(args.steps):
        flops += one_step((args.warmup + s_) % w.H)
    dt = time.perf_counter() - t0
    tf = flops / dt / 1e12
    line = {"metric": METRIC, "value": tf, "unit": "TFLOP/s", "n_gpus": int(os.environ.get("WORLD_SIZE", "1")),
            "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": bench_config(w, int(os.environ.get("WORLD_SIZE", "1"))),
            "cpu_baseline": {"value": tf, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                             "sample": "per step: one head's fp64 routing (permute, pool, scores, "
                                       "Top-p) and block-sparse attention of 2 query blocks"},
            "e2e": {"value": tf, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


SWEEP_PARITY_HEADS = range(0, 40, 5)


def run_sweep(args):
    """The 720p sweep (p x k_min x block size): one JSON line per config with its
    density, route and attention times and effective TFLOP/s (not the headline line),
    and, unless --no-cpu-baseline, its parity against the fp64 oracle: the masks of
    every query block of 8 heads (every fifth) and the outputs of each such head's
    tail block and heaviest row."""
    import block_sparse_attention_video_b200 as F
    _dist_setup(1)
    base = S.WORKLOADS["wan14b-720p"]
    q, k, v = S.make_qkv(base, device="cuda")
    stream = torch.cuda.current_stream()
    host = None if args.no_cpu_baseline else tuple(x.float().cpu().numpy() for x in (q, k, v))
    paths = {}
    for w in S.sweep_workloads():
        key = (w.block, w.tile)
        if key not in paths:
            paths.clear()
            torch.cuda.empty_cache()
            paths[key] = F.FVAttnPath(w.B, w.H, w.grid, w.tile, w.block, w.d, torch.bfloat16, w.p, w.k_min)
        path = paths[key]
        path.p, path.k_min = float(w.p), int(w.k_min)
        route_ms = _median_ms(lambda: path.route(q, k), stream, args.warmup, 3)
        F.fvattn_permute(v, path.vp, path.grid)
        attn_ms = _median_ms(lambda: path.attend(), stream, args.warmup, 3)
        if F.fvattn_workspace_status(path.ws_attn) != F.FVATTN_OK:
            raise RuntimeError("kernel status word set in the sweep")
        idx, cnt = path.kv_idx.cpu().numpy(), path.kv_cnt.cpu().numpy()
        eff = effective_flops(idx, cnt, w.N, w.block, w.d)
        hw = path.head_work.cpu().numpy().astype(np.float64)
        rec = {"sweep": w.name, "block": w.block, "p": w.p, "k_min": w.k_min,
               "density": float(cnt.mean() / path.nb), "route_ms": route_ms, "attention_ms": attn_ms,
               "effective_tflops": eff / (attn_ms * 1e-3) / 1e12,
               "head_work_max_over_mean": float(hw.max() / hw.mean())}
        if host is not None:
            mp, err, _, _, _, _ = oracle_check(w, *host, idx, cnt, path.op.float().cpu().numpy(),
                                               SWEEP_PARITY_HEADS, per_head=0, rng=np.random.default_rng(0))
            rec["mask_parity"] = mp
            rec["output_error"] = err
        print(json.dumps(rec), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("fvattn", "reference"), default="fvattn")
    ap.add_argument("--workload", default="wan14b-720p", choices=sorted(S.WORKLOADS))
    ap.add_argument("--block", type=int, choices=(64, 128), default=None,
                    help="run the workload with this block size (64: 1x8x8 tiles)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-diag", action="store_true", help="skip the GSRS block-importance diagnostic")
    ap.add_argument("--no-lvsa", action="store_true", help="skip the LVSA static-mask measurement")
    ap.add_argument("--no-hilbert", action="store_true", help="skip the Hilbert-order measurement")
    ap.add_argument("--no-fp8v", action="store_true", help="skip the E4M3-V attention measurement")
    ap.add_argument("--sweep", action="store_true",
                    help="print the 720p p x k_min x block-size sweep (one JSON line per config) instead")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    args = ap.parse_args(argv)
    if args.warmup < 3 and args.impl == "fvattn":
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    if args.sweep:
        return run_sweep(args)
    return run_reference(args) if args.impl == "reference" else run_fvattn(args)


if __name__ == "__main__":
    sys.exit(main())
