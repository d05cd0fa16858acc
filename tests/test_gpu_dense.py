"""Dense SwiGLU layers against the oracle ("Show HN: 遅いコンピュータで GLM 5.2
を実行する", 実装済みの主な機能, router bullet: the first three layers are
dense): n_routed = 0, top_k = 0 -- no router, every token through the shared
experts only -- on the persistent decode kernel (T <= 8), the tcgen05
grouped GEMMs and the CUDA-core grouped kernels.  Same bar as every layer:
bit-exact Q8_0(h) codes, outputs within 2e-4 * ||y_ref||_inf per token."""
import pytest

import synth
from tests.parity_util import GpuLayer, compare_forward

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _dense(**kw):
    c = dict(hidden=512, inter=256, n_routed=0, n_shared=1, top_k=0, n_group=1, topk_group=1,
             routed_scaling_factor=2.5, bits=4, seed=0, x="iid", tokens=4)
    c.update(kw)
    return c


@pytest.mark.parametrize("bits", [8, 4, 2])
@pytest.mark.parametrize("T", [1, 4, 37])
def test_dense_layer(bits, T):
    cfg = _dense(bits=bits, seed=300 + T + bits)
    gl = GpuLayer(cfg, max_tokens=max(T, 9))
    compare_forward(gl, synth.tokens(cfg, T=T, device=DEV))
    gl.close()


def test_dense_layer_two_experts_cuda_core_path(monkeypatch):
    monkeypatch.setenv("COLI_NO_TC", "1")
    cfg = _dense(n_shared=2, seed=331)
    gl = GpuLayer(cfg, max_tokens=40)
    compare_forward(gl, synth.tokens(cfg, T=40, device=DEV))
    gl.close()


def test_dense_layer_glm_hidden_size():
    """Hidden 6144 (the GLM-5.2 width), one token, intermediate 4096 (the
    pages give no intermediate size for the dense layers)."""
    cfg = _dense(hidden=6144, inter=4096, seed=332)
    gl = GpuLayer(cfg, max_tokens=1)
    for s in range(2):
        compare_forward(gl, synth.tokens(cfg, T=1, device=DEV, stream=s))
    gl.close()
