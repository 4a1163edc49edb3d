"""The device generator writes exactly the bytes of the host generator."""
import numpy as np
import pytest
import torch

import datagen as D

pytestmark = pytest.mark.gpu


def test_device_generator_matches_host():
    import datagen.gpu as G
    from tests._util import bf16_bits
    k = D.stream_key(11, D.TID_COMP, 2)
    t = G.normal_bf16_(torch.empty(3 * 100003, dtype=torch.bfloat16, device="cuda"), k, offset=777)
    assert np.array_equal(bf16_bits(t), D.normal_bf16(k, 3 * 100003, offset=777))
    k2 = D.stream_key(11, D.TID_KIDX, 0)
    t2 = G.int_bf16_(torch.empty(50000, dtype=torch.bfloat16, device="cuda"), k2, -8, 8, offset=5)
    assert np.array_equal(bf16_bits(t2), D.int_bf16(k2, 50000, -8, 8, offset=5))
    k3 = D.stream_key(11, D.TID_KIDX_FP4, 0)
    codes = torch.empty(300, 64, dtype=torch.uint8, device="cuda")
    scales = torch.empty(300, 8, dtype=torch.uint8, device="cuda")
    G.fp4_index_keys_(codes, scales, k3, row0=1000)
    hc, hs = D.fp4_index_keys_rows(k3, np.arange(1000, 1300), 128)
    assert np.array_equal(codes.cpu().numpy(), hc) and np.array_equal(scales.cpu().numpy(), hs)
