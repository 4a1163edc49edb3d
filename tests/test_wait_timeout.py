"""The device-side failure path: a bounded wait that runs out reports
DSV4KV_DEV_TIMEOUT through the status word, and the context stays usable
(a call right after it is still correct)."""
import numpy as np
import pytest
import torch

import compressed_sparse_kv_b200 as K
import datagen as D
from oracle import formats as OF
from oracle import indexer as OI

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_the_context_survives():
    import datagen.gpu as G
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    K.selftest_wait_timeout(status)
    torch.cuda.synchronize()
    assert int(status.item()) & K.DEV_TIMEOUT
    # the next call on the same context runs normally
    b, n, k = 2, 5000, 512
    kk, kq = D.stream_key(61, D.TID_KIDX, 0), D.stream_key(61, D.TID_QIDX, 0)
    keys = G.int_bf16_(torch.empty(b, n, 128, dtype=torch.bfloat16, device="cuda"), kk, -8, 8)
    q = G.int_bf16_(torch.empty(b, 128, dtype=torch.bfloat16, device="cuda"), kq, -8, 8)
    ws = K.new_workspace(K.index_topk_workspace_bytes(b, n, k))
    idx, _ = K.index_topk(q, K.Cache(0, keys, None, 128), n, k, ws=ws)
    torch.cuda.synchronize()
    assert K.workspace_status(ws) == 0
    for s in range(b):
        kr = OF.bf16_bits_to_f64(D.rows_int_bf16(kk, np.arange(s * n, (s + 1) * n), 128))
        qr = OF.bf16_bits_to_f64(D.rows_int_bf16(kq, np.array([s]), 128)[0])
        ref, _ = OI.index_topk(qr, kr, k)
        assert np.array_equal(idx[s].cpu().numpy(), ref)

