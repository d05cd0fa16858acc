"""coli_router_static, the routing entry point that allocates nothing.

Some callers cannot allocate device memory where they route (their memory is
already handed to a caching allocator or a fixed budget, or their loop cannot
take cudaMalloc's implicit synchronisation).  coli_router_static keeps its
scratch in a fixed array inside the library, so it needs no handle.  Its
result must equal the handle-based coli_router's, call after call, even
though every call reuses the same scratch.
"""
import numpy as np
import pytest
import torch

import synth
import quantized_expert_ffn_noaux_b200 as qe

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _handle(cfg, W, b, max_tokens):
    lc = synth.layer_cfg(cfg)
    lc.update(max_tokens=max_tokens)
    dummy = qe.Expert(*[(torch.zeros((cfg["inter"], cfg["hidden"] // 2), dtype=torch.uint8,
                                     device=DEV), torch.zeros(cfg["inter"], device=DEV))] * 3)
    return qe.MoELayer(lc, W, b, [dummy] * (cfg["n_routed"] + cfg["n_shared"]))


def test_router_static_matches_router_on_consecutive_calls():
    cfg = synth.workload("glm52_decode_int4_t1")
    W, b = synth.router(cfg, device=DEV)
    h = _handle(cfg, W, b, max_tokens=8)
    for call, T in enumerate((4, 1, 8)):
        x = synth.tokens(cfg, T=T, device=DEV, stream=100 + call)
        idx_ref, w_ref = h.router(x)
        idx, w = qe.router_static(synth.layer_cfg(cfg), W, b, x)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(idx.cpu().numpy(), idx_ref.cpu().numpy())
        np.testing.assert_allclose(w.cpu().numpy(), w_ref.cpu().numpy(), rtol=1e-6)
    h.close()


def test_router_static_rejects_sizes_beyond_its_scratch():
    cfg = synth.workload("glm52_decode_int4_t1")
    W, b = synth.router(cfg, device=DEV)
    x = synth.tokens(cfg, T=9, device=DEV)
    with pytest.raises(qe.ColiError) as ei:
        qe.router_static(synth.layer_cfg(cfg), W, b, x)
    assert ei.value.status == qe.COLI_EINVAL and "T <=" in str(ei.value)


def test_router_static_leaves_free_memory_unchanged():
    """After the first call (which looks up the fixed array's address), further
    calls with preallocated outputs take no device memory: the device's free
    memory, as the driver reports it, is the same before and after them."""
    cfg = synth.workload("glm52_decode_int4_t1")
    W, b = synth.router(cfg, device=DEV)
    x = synth.tokens(cfg, T=8, device=DEV, stream=7)
    k = cfg["top_k"]
    idx = torch.empty((8, k), dtype=torch.int32, device=DEV)
    w = torch.empty((8, k), dtype=torch.float32, device=DEV)
    lc = synth.layer_cfg(cfg)
    qe.router_static(lc, W, b, x, idx=idx, w=w)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for T in (8, 1, 5, 8):
        qe.router_static(lc, W, b, x[:T], idx=idx[:T], w=w[:T])
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0


def test_router_static_rejects_more_experts_than_its_scratch():
    cfg = synth.workload("glm52_decode_int4_t1", n_routed=1025, n_group=1, topk_group=1)
    W, b = synth.router(cfg, device=DEV)
    x = synth.tokens(cfg, T=1, device=DEV)
    with pytest.raises(qe.ColiError) as ei:
        qe.router_static(synth.layer_cfg(cfg), W, b, x)
    assert ei.value.status == qe.COLI_EINVAL and "1024" in str(ei.value)


def test_router_static_rejects_a_dense_layer():
    cfg = synth.workload("glm52_decode_int4_t1")
    W, b = synth.router(cfg, device=DEV)
    x = synth.tokens(cfg, T=1, device=DEV)
    lc = dict(synth.layer_cfg(cfg), n_routed=0, top_k=0, n_group=1, topk_group=1)
    with pytest.raises(qe.ColiError) as ei:
        qe.router_static(lc, W[:0], b[:0], x, idx=torch.empty((1, 1), dtype=torch.int32, device=DEV),
                         w=torch.empty((1, 1), device=DEV))
    assert ei.value.status == qe.COLI_EINVAL


def test_router_static_top_p_matches_router():
    cfg = dict(synth.workload("glm52_decode_int4_t1"), expert_top_p=0.7)
    W, b = synth.router(cfg, device=DEV)
    h = _handle(cfg, W, b, max_tokens=8)
    x = synth.tokens(cfg, T=8, device=DEV, stream=11)
    idx_ref, w_ref = h.router(x)
    idx, w = qe.router_static(synth.layer_cfg(cfg), W, b, x)
    torch.cuda.synchronize()
    assert (idx_ref < 0).any()
    np.testing.assert_array_equal(idx.cpu().numpy(), idx_ref.cpu().numpy())
    np.testing.assert_allclose(w.cpu().numpy(), w_ref.cpu().numpy(), rtol=1e-6)
    h.close()
