"""The FP8 -> per-row requantiser (coli_requant_fp8) against the oracle, bit
for bit ("Show HN: 遅いコンピュータで GLM 5.2 を実行する", 実装済みの主な機能,
offline-converter bullet: FP8 shards dequantised with 128 x 128 block scales,
then requantised into the engine's container)."""
import numpy as np
import pytest
import torch

import oracle
import quantized_expert_ffn_noaux_b200 as qe

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _fp8_weights(rows, K, block, seed):
    """Random e4m3 codes (no NaN codes) and log-normal block scales."""
    r = np.random.default_rng(seed)
    codes = r.integers(0, 256, size=(rows, K), dtype=np.uint8)
    codes[(codes & 0x7F) == 0x7F] ^= 0x01             # S.1111.111 (NaN) -> S.1111.110
    codes[0, :min(K, 48)] = 0x00                       # zeros at a row start
    if rows > 1:                                       # hand-picked codes, signed zero, extremes
        codes[1, :16] = [0x00, 0x80, 0x01, 0x81, 0x07, 0x08, 0x38, 0xB8, 0x7E, 0xFE,
                         0x30, 0x39, 0x40, 0x77, 0x78, 0x0F]
    if rows > 2:
        codes[2, :] = 0x00                             # an all-zero row: scale 0, codes 0
    scale = np.exp(r.normal(-6.0, 1.0, size=(-(-rows // block), -(-K // block)))).astype(np.float32)
    return codes, scale


@pytest.mark.parametrize("bits", [8, 4, 2])
@pytest.mark.parametrize("rows,K,block", [(1, 64, 128), (130, 256, 128), (300, 6144, 128),
                                          (2048, 6144, 128), (6144, 2048, 128), (96, 192, 64)])
def test_requant_fp8_bitexact(bits, rows, K, block):
    codes, scale = _fp8_weights(rows, K, block, seed=rows * 7 + K + bits)
    c, s = qe.requant_fp8(torch.from_numpy(codes).to(DEV), torch.from_numpy(scale).to(DEV), bits,
                          block=block)
    co, so = oracle.requant_fp8(codes, scale, bits, block=block)
    np.testing.assert_array_equal(s.cpu().numpy(), so)
    np.testing.assert_array_equal(c.cpu().numpy(), co)


def test_requant_fp8_rejects_bad_arguments():
    w = torch.zeros((4, 64), dtype=torch.uint8, device=DEV)
    sc = torch.ones((1, 1), dtype=torch.float32, device=DEV)
    for bits, block, K in ((3, 128, 64), (4, 100, 64), (4, 0, 64), (2, 128, 32)):
        ww = w[:, :K]
        with pytest.raises(qe.ColiError) as ei:
            qe.requant_fp8(ww, sc, bits, block=block)
        assert ei.value.status == qe.COLI_EINVAL
