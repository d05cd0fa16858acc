"""Expert parallelism on one GPU: "virtual ranks" -- handles over the same
weights, each computing one contiguous range of routed experts (rank 0 also
the shared experts) -- whose fp64 partial outputs are summed in rank order
through coli_combine_partials.  The result must meet the oracle's bar like
any forward, equal the single-handle forward to within the association of
the fp64 sum, and equal it bit for bit when one rank holds everything.
(Across GPUs the partials travel by NCCL all-gather; that exchange is
covered by the gloo tests on the CPU.)"""
import numpy as np
import pytest
import torch

import synth
import quantized_expert_ffn_noaux_b200 as qe
from tests.parity_util import GpuLayer, compare_forward

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _cfg(**kw):
    c = dict(hidden=512, inter=256, n_routed=16, n_shared=1, top_k=3, n_group=4, topk_group=2,
             routed_scaling_factor=2.5, bits=4, seed=0, x="iid", tokens=4)
    c.update(kw)
    return c


def _ranks(gl, world, max_tokens):
    lc = synth.layer_cfg(gl.cfg)
    lc["max_tokens"] = max_tokens
    hs = []
    for r in range(world):
        h = qe.MoELayer(lc, gl.Wr, gl.bias, gl.experts)
        lo, hi = qe.expert_range(gl.cfg["n_routed"], r, world)
        h.set_experts(lo, hi, own_shared=(r == 0))
        hs.append(h)
    return hs


@pytest.mark.parametrize("T", [1, 4, 37])
@pytest.mark.parametrize("world", [1, 2, 3])
def test_expert_parallel_partials(T, world):
    """T = 1 and 4 take the persistent decode kernel, T = 37 the tcgen05
    grouped GEMMs; with 3 ranks and T = 1 some rank owns none of the token's
    experts."""
    cfg = _cfg(seed=200 + T + world)
    gl = GpuLayer(cfg, max_tokens=max(T, 9))
    x = synth.tokens(cfg, T=T, device=DEV)
    y_np, _ = compare_forward(gl, x)          # the single handle meets the oracle's bar
    y_full = torch.from_numpy(y_np).to(DEV)
    hs = _ranks(gl, world, max(T, 9))
    parts = torch.stack([h.forward_partial(x) for h in hs])
    y = qe.combine_partials(parts)
    torch.cuda.synchronize()
    if world == 1:
        assert torch.equal(y, y_full)
    else:
        ref = y_full.double()
        err = (y.double() - ref).abs().max(dim=1).values
        assert torch.all(err <= 1e-6 * ref.abs().max(dim=1).values)
    # repeated calls are bit-identical (fixed order of the fp64 sums)
    y2 = qe.combine_partials(torch.stack([h.forward_partial(x) for h in hs]))
    assert torch.equal(y, y2)
    for h in hs:
        h.close()
    gl.close()


def test_expert_parallel_cuda_core_grouped_path(monkeypatch):
    """The CUDA-core grouped kernels (COLI_NO_TC=1) with two ranks."""
    monkeypatch.setenv("COLI_NO_TC", "1")
    cfg = _cfg(seed=230)
    gl = GpuLayer(cfg, max_tokens=40)
    x = synth.tokens(cfg, T=40, device=DEV)
    y_np, _ = compare_forward(gl, x)
    hs = _ranks(gl, 2, 40)
    y = qe.combine_partials(torch.stack([h.forward_partial(x) for h in hs]))
    ref = torch.from_numpy(y_np).double()
    err = (y.cpu().double() - ref).abs().max(dim=1).values
    assert torch.all(err <= 1e-6 * ref.abs().max(dim=1).values)
    for h in hs:
        h.close()
    gl.close()


def test_expert_range_is_validated():
    cfg = _cfg(seed=231)
    gl = GpuLayer(cfg, max_tokens=4)
    with pytest.raises(qe.ColiError):
        gl.handle.set_experts(3, 2)
    with pytest.raises(qe.ColiError):
        gl.handle.set_experts(0, cfg["n_routed"] + 1)
    gl.close()
