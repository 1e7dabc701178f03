"""The hot path under CUDA-graph capture.

Every entry point is asynchronous on the caller's stream, allocates nothing
and never synchronises the host (the split sizes stay on the device), so a
whole step -- offsets, the three bf16 GEMMs, the MXFP8 casts and the three
MXFP8 GEMMs -- can be captured once and replayed.  Replays must reproduce the
eager results bit for bit, follow new split sizes written into the captured
device buffer, and (the weight-cast ``noop`` use of ``grouped_linear.py``'s
quantizers, PR #3224 "Improve device-init grouped linear module") skip a
cast whose status word is set.
"""
import numpy as np
import pytest
import torch

from grouped_gemm_splits_b200 import gl, synth
from oracle import gl_oracle as orc
from tests.gpu_util import f64

pytestmark = pytest.mark.gpu


def _buffers(G, M, N, K, m, seed):
    d = {k: v.cuda() for k, v in synth.operands(G, M, N, K, seed=seed, bias=True).items()}
    d["m"] = torch.tensor(m, dtype=torch.int64, device="cuda")
    d["off"] = torch.empty(G + 1, dtype=torch.int64, device="cuda")
    d["st"] = torch.zeros(1, dtype=torch.int32, device="cuda")
    d["y"] = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    d["dx"] = torch.empty(M, K, dtype=torch.bfloat16, device="cuda")
    d["ymx"] = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    d["dxmx"] = torch.empty(M, K, dtype=torch.bfloat16, device="cuda")
    d["mg0"] = d["main_grad"].clone()
    d["mgmx"] = torch.zeros(G, N, K, device="cuda")
    d["qx"], d["qdy"], d["qw"] = {}, {}, {}
    return d


def _step(d, M):
    gl.gl_offsets(d["m"], M, M, d["off"], d["st"])
    gl.gl_fwd(d["x"], d["w"], d["bias"], d["off"], d["st"], d["y"])
    gl.gl_dgrad(d["dy"], d["w"], d["off"], d["st"], d["dx"])
    gl.gl_wgrad(d["x"], d["dy"], d["off"], d["st"], d["main_grad"], accumulate=True)
    gl.group_quantize_mxfp8(d["x"], d["off"], rowwise=True, colwise=True, status=d["st"], out=d["qx"], mma_scales=True)
    gl.group_quantize_mxfp8(d["dy"], d["off"], rowwise=True, colwise=True, status=d["st"], out=d["qdy"],
                            mma_scales=True)
    gl.group_quantize_mxfp8(d["w"], rowwise=True, colwise=True, out=d["qw"], mma_scales=True)
    G, N, K = d["w"].shape
    gl.gl_fwd_mxfp8(d["qx"]["codes_r"], d["qx"]["scales_r"], d["qw"]["codes_r"].view(G, N, K), d["qw"]["scales_r"],
                    d["bias"], d["off"], d["st"], d["ymx"])
    gl.gl_dgrad_mxfp8(d["qdy"]["codes_r"], d["qdy"]["scales_r"], d["qw"]["codes_c"].view(G, N, K),
                      d["qw"]["scales_c"], d["off"], d["st"], d["dxmx"])
    gl.gl_wgrad_mxfp8(d["qx"]["codes_c"], d["qx"]["scales_c"], d["qdy"]["codes_c"], d["qdy"]["scales_c"], d["off"],
                      d["st"], d["mgmx"], accumulate=False)


def _snapshot(d):
    return {k: d[k].clone() for k in ("y", "dx", "main_grad", "ymx", "dxmx", "mgmx")}


def test_graph_replay_matches_eager():
    G, N, K = 4, 256, 256
    m = [0, 200, 57, 255]
    M = sum(m)
    eager = _buffers(G, M, N, K, m, seed=11)
    _step(eager, M)
    torch.cuda.synchronize()
    ref = _snapshot(eager)

    d = _buffers(G, M, N, K, m, seed=11)
    _step(d, M)  # warm: allocations of the cast outputs happen outside the capture
    d["main_grad"].copy_(d["mg0"])
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(graph, stream=s):
            _step(d, M)
    d["main_grad"].copy_(d["mg0"])
    graph.replay()
    torch.cuda.synchronize()
    got = _snapshot(d)
    for k in ref:
        assert torch.equal(got[k].view(torch.int32) if got[k].dtype == torch.float32 else got[k].view(torch.int16),
                           ref[k].view(torch.int32) if ref[k].dtype == torch.float32 else ref[k].view(torch.int16)), k
    assert int(d["st"].item()) == 0

    # new split sizes written into the captured device buffer are followed
    m2 = [100, 100, 212, 100]
    d["m"].copy_(torch.tensor(m2, device="cuda"))
    graph.replay()
    eager2 = _buffers(G, M, N, K, m2, seed=11)
    _step(eager2, M)
    torch.cuda.synchronize()
    assert torch.equal(d["y"].view(torch.int16), eager2["y"].view(torch.int16))
    assert torch.equal(d["ymx"].view(torch.int16), eager2["ymx"].view(torch.int16))
    del graph


def test_graph_weight_cast_noop_flag():
    """A captured weight cast into caller-owned (reused) buffers skips its
    work on replays where its status word (used as the noop flag) is non-zero,
    and once the flag is cleared writes the oracle's codes and scales into
    those same buffers."""
    G, N, K = 2, 128, 256
    w = torch.randn(G, N, K, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16).cuda()
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    q = {}
    gl.group_quantize_mxfp8(w, rowwise=True, colwise=True, status=flag, out=q, mma_scales=True)
    torch.cuda.synchronize()
    first = {k: v.clone() for k, v in q.items()}
    s = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(graph, stream=s):
            gl.group_quantize_mxfp8(w, rowwise=True, colwise=True, status=flag, out=q, mma_scales=True)
    for v in q.values():
        v.fill_(0xAB)
    flag.fill_(1)
    graph.replay()
    torch.cuda.synchronize()
    assert all(bool((v == 0xAB).all().item()) for v in q.values())
    flag.fill_(0)
    graph.replay()
    torch.cuda.synchronize()
    assert int(flag.item()) == 0
    # what the replay wrote into the reused caller buffers is the oracle's
    # cast of W (G equal members), scales read back through the MMA layout
    src = f64(w.reshape(G * N, K))
    cr, sr = orc.quantize_rowwise(src)
    cc, sc = orc.quantize_colwise(src, [N] * G)
    assert np.array_equal(q["codes_r"].cpu().numpy().reshape(G * N, K), cr)
    assert np.array_equal(q["scales_r"].cpu().numpy()[orc.mma_offsets_rowwise(G * N, K)], sr)
    assert np.array_equal(q["codes_c"].cpu().numpy().reshape(G * N, K), cc)
    assert np.array_equal(q["scales_c"].cpu().numpy()[orc.mma_offsets_colwise([N] * G, K)], sc)
    for k in ("codes_r", "codes_c"):
        assert torch.equal(q[k], first[k]), k
    del graph
