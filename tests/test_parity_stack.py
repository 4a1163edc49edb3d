"""The 61-layer stack step's layers at their full size (B = 1, t = 2^20,
H = 64) against the float64 oracle, built and launched exactly as the bench
times them (bench.Layer: the same seeded caches, shared index and decode
workspaces, one CUDA graph over the layers).

* c128a layer: dense attention over 8191 entries + 128 window rows; with one
  sequence the decode splits its 130 tiles over 130 CTAs and the many-split
  merge (decode_combine_wide) joins them.
* c4a layer: the GPU top-512 of 262112 indexer keys (bit-exact against the
  oracle's), then the sparse decode of the selected rows + window (10 tiles,
  10 splits).
* a three-layer step (c128a, c4a, c128a) captured in one CUDA graph and
  replayed, every layer's output checked.

[P1] "c128a (the aggressive scheme)", "c4a (the milder scheme)" and the layer
stack (30 c4a + 31 c128a layers of a 1M-token sequence)."""
import numpy as np
import pytest
import torch

import bench
import datagen as D
from datagen import workloads as WL
from oracle import attention as OA
from oracle import formats as OF
from oracle import indexer as OI
from tests._util import assert_close, to_f64

pytestmark = pytest.mark.gpu
T = 1 << 20
SEED = 4242
SCALE = 512 ** -0.5


def _layer(layer_id, shared=None):
    return bench.Layer(WL.stack_layer_kind(layer_id), 1, T, 64, SEED, 1, layer_id=layer_id, shared=shared)


def _expected(L, layer_id):
    """(oracle indices or None, oracle output [H][512]) of sequence 0 of a bench layer."""
    keys = WL.keys_for(SEED, layer_id)  # replica 0 uses the layer's own keys
    q = OF.bf16_bits_to_f64(D.rows_normal_bf16(keys["q"], np.arange(64), 512))
    win = OF.bf16_bits_to_f64(D.rows_normal_bf16(keys["win"], np.arange(L.window), 512))
    if L.kind == "c128a":
        comp = OF.bf16_bits_to_f64(D.rows_normal_bf16(keys["comp"], np.arange(L.n), 512))
        return None, OA.dense_decode(q[None], comp[None], win[None], T, SCALE)[0]
    kr = OF.bf16_bits_to_f64(D.rows_int_bf16(keys["kidx"], np.arange(L.n), 128))
    qi = OF.bf16_bits_to_f64(D.rows_int_bf16(keys["qidx"], np.array([0]), 128)[0])
    idx, cnt = OI.index_topk(qi, kr, L.k)
    sel = idx[:cnt].astype(np.int64)
    comp = np.zeros((L.n, 512))
    comp[sel] = OF.bf16_bits_to_f64(D.rows_normal_bf16(keys["comp"], sel, 512))
    return idx, OA.sparse_decode(q[None], comp[None], win[None], idx[None], T, SCALE)[0]


def _check(L, layer_id, out, idx=None):
    ref_idx, ref = _expected(L, layer_id)
    if ref_idx is not None:
        assert np.array_equal(idx.cpu().numpy()[0], ref_idx), f"layer {layer_id}: top-k differs from the oracle"
    assert_close(to_f64(out)[0], ref, what=f"layer {layer_id} ({L.kind})")


@pytest.mark.parametrize("layer_id", [0, 1])     # layer 0 is c128a, layer 1 is c4a
def test_stack_layer_at_full_size(layer_id):
    L = _layer(layer_id)
    L.step(0)
    torch.cuda.synchronize()
    assert L.K.workspace_status(L.ws_dec) == 0
    if L.kind == "c4a":
        assert L.K.workspace_status(L.ws_idx) == 0
    _check(L, layer_id, L.out, L.idx.clone() if L.kind == "c4a" else None)


def test_three_layer_stack_step_in_a_graph():
    shared = {}
    layers = [_layer(l, shared) for l in range(3)]
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        for L in layers:                 # eager warm-up, as the bench does
            L.step(0)
    stream.synchronize()
    for L in layers:
        L.out.zero_()
    g = torch.cuda.CUDAGraph()
    idx_after = {}
    with torch.cuda.graph(g, stream=stream):
        for i, L in enumerate(layers):
            if L.kind == "c4a":
                L.index(0)
                idx_after[i] = L.idx.clone()  # the shared index buffer, as this layer's decode read it
            L.decode(0)
    with torch.cuda.stream(stream):
        g.replay()
        g.replay()
    stream.synchronize()
    for i, L in enumerate(layers):
        _check(L, i, L.out, idx_after.get(i))
    assert layers[0].K.workspace_status(shared["ws_dec"]) == 0
    del g
