"""dsv4kv_index_topk_noalloc: the allocation-free indexer variant for callers
that cannot allocate device memory (e.g. a serving engine whose memory
manager owns all of HBM).  It must return exactly what dsv4kv_index_topk
returns with a caller workspace, call after call, since the static scratch
keeps the previous call's contents.  This file is collected last on purpose."""
import numpy as np
import pytest
import torch

import compressed_sparse_kv_b200 as K
import datagen as D

pytestmark = pytest.mark.gpu


def _inputs(seed, b, n):
    import datagen.gpu as G
    keys = G.int_bf16_(torch.empty(b, n, 128, dtype=torch.bfloat16, device="cuda"), D.stream_key(seed, D.TID_KIDX))
    q = G.int_bf16_(torch.empty(b, 128, dtype=torch.bfloat16, device="cuda"), D.stream_key(seed, D.TID_QIDX))
    return q, keys


def test_noalloc_matches_workspace_version_on_consecutive_calls():
    assert K.lib().dsv4kv_index_topk_noalloc_max_scratch_bytes() == 8 << 20
    for call, (b, n, k) in enumerate([(32, 32736, 512), (3, 5000, 64)]):
        q, keys = _inputs(40 + call, b, n)
        cache = K.Cache(0, keys, None, 128)
        ref_idx, ref_cnt = K.index_topk(q, cache, n, k)
        got_idx, got_cnt = K.index_topk_noalloc(q, cache, n, k)
        torch.cuda.synchronize()
        assert torch.equal(got_idx, ref_idx), f"call {call}: indices differ"
        assert torch.equal(got_cnt, ref_cnt), f"call {call}: counts differ"


def test_noalloc_rejects_sizes_above_the_static_maximum():
    q, keys = _inputs(9, 64, 40000)          # needs more than 8 MiB of scratch
    with pytest.raises(K.Dsv4kvError) as e:
        K.index_topk_noalloc(q, K.Cache(0, keys, None, 128), 40000, 512)
    assert e.value.status == 2 and "static maximum" in str(e.value)
