"""GPU: HostPipeline (pinned host inputs and outputs, copies of neighbouring calls
overlapping the current call's kernels, optionally per head range on separate
streams) gives, call by call, exactly the output of FVAttnPath on device inputs
(the kernels are deterministic per work unit); a
whole call captured in a CUDA graph (bf16 or E4M3 V) replays to the eager result."""

import pytest
import torch

import synthetic as S

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import block_sparse_attention_video_b200 as F


@pytest.mark.parametrize("head_groups", [1, 3, 12])   # 12: one head per range
@pytest.mark.parametrize("dense", [False, True])
def test_host_pipeline_matches_per_call_results(dense, head_groups):
    w = S.WORKLOADS["wan1.3b-480p"]
    calls = [S.make_qkv(w.replace(seed=w.seed + 100 * i), device="cuda") for i in range(3)]
    path = F.FVAttnPath(w.B, w.H, w.grid, w.tile, w.block, w.d, torch.bfloat16, w.p, w.k_min)
    want = [path(q, k, v, dense=dense).clone() for (q, k, v) in calls]
    host_in = [tuple(x.cpu().pin_memory() for x in qkv) for qkv in calls]
    host_out = [torch.empty(want[0].shape, dtype=want[0].dtype).pin_memory() for _ in calls]
    pipe = F.HostPipeline(path, dense=dense, head_groups=head_groups)
    pipe.run(host_in, host_out)
    torch.cuda.synchronize()
    for _, _, sub in pipe.parts:
        assert F.fvattn_workspace_status(sub.ws_attn) == F.FVATTN_OK
        if not dense:                     # a dense call does not route
            assert F.fvattn_workspace_status(sub.ws_route) == F.FVATTN_OK
    for i in range(len(calls)):
        assert torch.equal(host_out[i], want[i].cpu()), i
    # a second run reuses the same slots
    host_out2 = [torch.zeros_like(h) for h in host_out]
    host_out2 = [h.pin_memory() for h in host_out2]
    pipe.run(host_in[::-1], host_out2)
    torch.cuda.synchronize()
    for i in range(len(calls)):
        assert torch.equal(host_out2[i], want[::-1][i].cpu()), i


@pytest.mark.parametrize("v_format", ["bf16", "e4m3"])
@pytest.mark.parametrize("dense", [False, True])
def test_cuda_graph_replay_matches_eager(dense, v_format):
    w = S.WORKLOADS["wan1.3b-480p"]
    q, k, v = S.make_qkv(w, device="cuda")
    path = F.FVAttnPath(w.B, w.H, w.grid, w.tile, w.block, w.d, torch.bfloat16, w.p, w.k_min,
                        v_format=v_format)
    out = torch.empty_like(q)
    graph, res = path.capture_graph(q, k, v, dense=dense, out=out)
    for shift in (7, 19):
        q2, k2, v2 = S.make_qkv(w.replace(seed=w.seed + shift), device="cuda")
        want = path(q2, k2, v2, dense=dense).clone()
        q.copy_(q2)
        k.copy_(k2)
        v.copy_(v2)
        res.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert F.fvattn_workspace_status(path.ws_attn) == F.FVATTN_OK
        assert torch.equal(res, want), shift
