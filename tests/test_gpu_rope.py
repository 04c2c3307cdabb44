"""GPU parity of the RoPE switches: rotary width, pair style and block-position scale.

The pages ask for RoPE at the block position ("Part 10", section "QSA indexer") without
fixing the pairing, the rotary width or the position scale. The library's default is the
NeoX half-split over all dims with block b at token 4b; the layer config can select the
other readings, and each must match the oracle with the same switches, in the pooled
cache (bulk and fused decode updates, incremental == full rebuild) and in the scores and
selection of the indexer scan.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import qsa_oracle as O
from tests import gpu_harness as H

pytestmark = pytest.mark.gpu

# (workload, switches): d_idx 64 on "tiny", 128 on the pages' layer shape
VARIANTS = [
    ("tiny", dict(rope_interleaved=True)),
    ("tiny", dict(rope_dims=32)),
    ("tiny", dict(rope_dims=16, rope_interleaved=True, rope_pos_stride=1)),
    ("tiny", dict(rope_pos_stride=1)),
    ("tiny", dict(rope_pos_offset=3)),
    ("tiny", dict(rope_dims=48, rope_pos_stride=2, rope_pos_offset=5)),
    ("ctx64k", dict(rope_dims=96)),
    ("ctx64k", dict(rope_interleaved=True, rope_pos_stride=1)),
    ("ctx64k", dict(rope_dims=64, rope_interleaved=True, rope_pos_offset=2)),
]
IDS = [f"{w}-" + "-".join(f"{k[5:]}{int(v)}" for k, v in sw.items()) for w, sw in VARIANTS]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    H.ensure_library()


def _setup(wl_name, sw, max_ctx):
    import sparse_attention_decode_02_b200 as Q
    wl = synth.workload(wl_name)
    qsa = Q.Qsa(H.config_of(wl, max_ctx=max_ctx, **sw))
    return wl, qsa, H.GpuLayer(qsa), O.QsaShape.of(wl, **sw)


@pytest.mark.parametrize("wl_name,sw", VARIANTS, ids=IDS)
def test_pooled_cache_with_rope_switches(wl_name, sw):
    n0 = 1023
    wl, qsa, g, shape = _setup(wl_name, sw, max_ctx=1040)
    pre = synth.prefill_tokens(wl, 0, n0)
    g.append(pre["k"], pre["v"], pre["idx"])
    g.update()                                   # bulk pooling kernel
    idx = [pre["idx"]]
    for step in range(9):                        # fused decode kernel, across two block ends
        st = synth.step_inputs(wl, 0, step)
        qsa.decode_append(0, H.to_dev(st["k"]), H.to_dev(st["v"]), H.to_dev(st["idx"]))
        idx.append(st["idx"][None])
    n = n0 + 9
    assert g.state() == (n, n // 4, 0)
    raw = np.concatenate(idx)
    inc = g.pooled_rows(0, n // 4)
    H.assert_pooled_close(inc, O.pooled_cache_full(raw, n, shape))
    qsa.invalidate_pooled_cache(0, 0)
    g.buf["pooled_cache"].zero_()
    g.update()
    np.testing.assert_array_equal(g.pooled_rows(0, n // 4), inc)


@pytest.mark.parametrize("wl_name,sw", VARIANTS, ids=IDS)
@pytest.mark.parametrize("n", [4 * 700 + 2, 4 * 3001])
def test_scores_and_selection_with_rope_switches(wl_name, sw, n):
    wl, qsa, g, shape = _setup(wl_name, sw, max_ctx=(n + 2 + 3) // 4 * 4)
    pooled = synth.random_pooled(wl, 0, n // 4, salt=n + 17)
    g.buf["pooled_cache"][: len(pooled)] = H.to_dev(pooled)
    qsa.restore_layer(0, n, n // 4)
    st = synth.step_inputs(wl, 0, 3)
    g.index_topk(st["q_idx"], st["w"])
    res = g.fetch()
    ref = O.block_scores(pooled, st["q_idx"], st["w"], n, shape)
    assert np.abs(res["scores"][: n // 4] - ref).max() <= H.SCORE_REL * np.abs(ref).max()
    H.selection_mismatch(res["sel"], ref, shape.k_blocks, H.TIE_GAP_REL)
    # switches that change the query's rotation change the scores of a fixed pooled table
    # (the offset moves only the blocks, so it shows in the pooled rows instead)
    if set(sw) - {"rope_pos_offset"}:
        dflt = O.block_scores(pooled, st["q_idx"], st["w"], n, O.QsaShape.of(wl))
        assert np.abs(dflt - ref).max() > 100 * H.SCORE_REL * np.abs(ref).max()
    assert g.state()[2] == 0
