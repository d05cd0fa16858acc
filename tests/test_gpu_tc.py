"""Tensor-core grouped path (many tokens) vs the oracle, through the C ABI.

Shapes whose hidden and intermediate sizes are whole stages of 8 Q8_0 blocks
take the tcgen05 grouped GEMMs (gate/up + SwiGLU + Q8_0(h), then down, then
the combine).  The bar is the one of every parity test: bit-exact routing of
decidable tokens and Q8_0(h) codes and scales, fp32 outputs within
2e-4 * ||y_ref||_inf per token.  Token counts are chosen so that the
per-expert token lists end in ragged 32-token tiles.
"""
import pytest

import synth
from tests.parity_util import GpuLayer, compare_forward

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _cfg(**kw):
    c = dict(hidden=512, inter=256, n_routed=16, n_shared=1, top_k=3, n_group=4, topk_group=2,
             routed_scaling_factor=2.5, bits=4, seed=0, x="iid", tokens=4)
    c.update(kw)
    return c


def _ran_tensor_cores(gl, x):
    gl.handle.profile(True)
    gl.handle.forward(x)
    names = gl.handle.profile_read()
    gl.handle.profile(False)
    return "gateup_tc" in names and "down_tc" in names


@pytest.mark.parametrize("bits", [8, 4, 2])
@pytest.mark.parametrize("T", [9, 37, 200])
def test_grouped_tensor_core_path(bits, T):
    cfg = _cfg(bits=bits, seed=300 + T + bits)
    gl = GpuLayer(cfg, max_tokens=T)
    x = synth.tokens(cfg, T=T, device=DEV)
    assert _ran_tensor_cores(gl, x)
    compare_forward(gl, x)
    gl.close()


def test_grouped_tensor_core_two_shared_experts_long_rows():
    """Two shared experts (every token in both: 4 ragged tiles each) and a
    hidden size of 3 stages."""
    cfg = _cfg(hidden=768, inter=512, n_shared=2, n_routed=8, top_k=2, n_group=2, topk_group=1,
               seed=41)
    T = 100
    gl = GpuLayer(cfg, max_tokens=T)
    x = synth.tokens(cfg, T=T, device=DEV)
    assert _ran_tensor_cores(gl, x)
    compare_forward(gl, x)
    gl.close()


def test_grouped_tensor_core_repeat_is_bit_identical():
    cfg = _cfg(seed=43)
    gl = GpuLayer(cfg, max_tokens=64)
    x = synth.tokens(cfg, T=64, device=DEV)
    a = gl.handle.forward(x).clone()
    b = gl.handle.forward(x).clone()
    assert (a == b).all()
    assert gl.handle.device_status() == 0
    gl.close()


def test_cuda_core_grouped_path_on_tensor_core_shapes(monkeypatch):
    """COLI_NO_TC=1 (read when the handle is created) keeps the CUDA-core
    grouped kernels on shapes the tensor-core path would take: both many-token
    paths meet the same bar on the same inputs."""
    monkeypatch.setenv("COLI_NO_TC", "1")
    cfg = _cfg(bits=4, seed=47)
    gl = GpuLayer(cfg, max_tokens=40)
    x = synth.tokens(cfg, T=40, device=DEV)
    assert not _ran_tensor_cores(gl, x)
    compare_forward(gl, x)
    gl.close()
