"""dsv4kv_index_topk_noalloc: the allocation-free indexer variant for callers
that cannot allocate device memory (e.g. a serving engine whose memory
manager owns all of HBM).  It must return exactly what dsv4kv_index_topk
returns with a caller workspace, call after call, since the static scratch
keeps the previous call's contents, and its status word must read zero after
good calls.  This file is collected last on purpose."""
import numpy as np
import pytest
import torch

import compressed_sparse_kv_b200 as K
import datagen as D

pytestmark = pytest.mark.gpu


def _inputs(seed, b, n, fmt):
    import datagen.gpu as G
    q = G.int_bf16_(torch.empty(b, 128, dtype=torch.bfloat16, device="cuda"), D.stream_key(seed, D.TID_QIDX))
    if fmt == K.BF16:
        keys = G.int_bf16_(torch.empty(b, n, 128, dtype=torch.bfloat16, device="cuda"), D.stream_key(seed, D.TID_KIDX))
        return q, K.Cache(K.BF16, keys, None, 128)
    codes = torch.empty(b, n, 64, dtype=torch.uint8, device="cuda")
    scales = torch.empty(b, n, 8, dtype=torch.uint8, device="cuda")
    G.fp4_index_keys_(codes, scales, D.stream_key(seed, D.TID_KIDX_FP4))
    return q, K.Cache(K.FP4_E2M1_G16, codes, scales, 128)


@pytest.mark.parametrize("fmt", [K.BF16, K.FP4_E2M1_G16])
def test_noalloc_matches_workspace_version_on_consecutive_calls(fmt):
    assert K.lib().dsv4kv_index_topk_noalloc_max_scratch_bytes() == 8 << 20
    K.index_topk_noalloc_status(clear=True)
    # a large call, a small one, a larger one after it (stale counters beyond the
    # small call's prefix would show), a call with n <= k, and the first shape again
    shapes = [(32, 32736, 512), (3, 5000, 64), (20, 9000, 300), (4, 400, 512), (32, 32736, 512)]
    stream = torch.cuda.Stream()
    for call, (b, n, k) in enumerate(shapes):
        q, cache = _inputs(40 + call, b, n, fmt)
        ref_idx, ref_cnt = K.index_topk(q, cache, n, k)
        s = stream if call % 2 else None        # every other call on a non-default stream
        if s is not None:
            s.wait_stream(torch.cuda.current_stream())
        got_idx, got_cnt = K.index_topk_noalloc(q, cache, n, k, stream=s)
        torch.cuda.synchronize()
        assert torch.equal(got_idx, ref_idx), f"call {call}: indices differ"
        assert torch.equal(got_cnt, ref_cnt), f"call {call}: counts differ"
    assert K.index_topk_noalloc_status(clear=True) == 0


def test_noalloc_rejects_sizes_above_the_static_maximum():
    q, cache = _inputs(9, 64, 40000, K.BF16)          # needs more than 8 MiB of scratch
    with pytest.raises(K.Dsv4kvError) as e:
        K.index_topk_noalloc(q, cache, 40000, 512)
    assert e.value.status == 2 and "static maximum" in str(e.value)
