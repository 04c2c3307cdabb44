"""GPU parity of the CUDA-core indexer scan (layer option scan_kind = QSA_SCAN_CUDA_CORES).

The scan scores the current indexer query against every completed block ("Part 10",
section "QSA indexer"); the library computes the dots either on the tensor cores (the
default) or on the CUDA cores with an f32 query. Both must give the oracle's scores on
identical f16 pooled tables within the score tolerance, and the selection bit-exact up to
near-ties, for every head count and key width the kernels are built for.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import qsa_oracle as O
from tests import gpu_harness as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    H.ensure_library()


def _qsa(wl, max_ctx, scan_kind):
    import sparse_attention_decode_02_b200 as Q
    cfg = H.config_of(wl, max_ctx=max_ctx)
    cfg.scan_kind = scan_kind
    return Q.Qsa(cfg)


# (workload, overrides, n): d 64 and 128 with 1..16 heads (lanes per row 8 and 16, so both
# the more-heads-than-lanes and the fewer-heads-than-lanes reductions), ragged chunk tails
CASES = [
    ("tiny", {}, 1027),
    ("tiny", dict(n_idx_heads=16), 4 * 300 + 2),
    ("tiny", dict(n_idx_heads=1), 4 * 77 + 3),
    ("ctx64k", dict(n_idx_heads=2), 4 * 4000 + 1),
    ("ctx64k", dict(n_idx_heads=8), 4 * 5003),
    ("ctx64k", {}, 61790),
    ("ctx256k_12l", {}, 255182),
]


@pytest.mark.parametrize("wl_name,over,n", CASES, ids=[f"{c[0]}-H{c[1].get('n_idx_heads', 'def')}-{c[2]}"
                                                       for c in CASES])
def test_cuda_core_scan_matches_oracle_and_tensor_core_scan(wl_name, over, n):
    import sparse_attention_decode_02_b200 as Q
    wl = synth.workload(wl_name, **over)
    shape = O.QsaShape.of(wl)
    pooled = synth.random_pooled(wl, 0, n // 4, salt=n)
    st = synth.step_inputs(wl, 0, 0)
    ref_scores = O.block_scores(pooled, st["q_idx"], st["w"], n, shape)
    got = {}
    for kind in (Q.QSA_SCAN_CUDA_CORES, Q.QSA_SCAN_TENSOR):
        qsa = _qsa(wl, ((n + 3) // 4) * 4 + 4, kind)
        g = H.GpuLayer(qsa)
        g.buf["pooled_cache"][: len(pooled)] = H.to_dev(pooled)
        qsa.restore_layer(0, n, n // 4)
        g.index_topk(st["q_idx"], st["w"])
        res = g.fetch()
        gs = res["scores"][: n // 4]
        assert np.abs(gs - ref_scores).max() <= H.SCORE_REL * np.abs(ref_scores).max(), kind
        H.selection_mismatch(res["sel"], ref_scores, shape.k_blocks, H.TIE_GAP_REL)
        assert g.state()[2] == 0
        got[kind] = gs
    # the two scans agree with each other to the same tolerance
    cc, tc = got[Q.QSA_SCAN_CUDA_CORES], got[Q.QSA_SCAN_TENSOR]
    assert np.abs(cc - tc).max() <= 2 * H.SCORE_REL * np.abs(ref_scores).max()


def test_cuda_core_scan_decode_chain_and_stale_cache():
    """qsa_decode_step on a CUDA-core layer (append + pooled update, scan, selection,
    attention) against the oracle's chain; a stale pooled cache is refused."""
    import sparse_attention_decode_02_b200 as Q
    wl = synth.workload("tiny")
    n0 = 1018
    qsa = _qsa(wl, (n0 + 16 + 3) // 4 * 4, Q.QSA_SCAN_CUDA_CORES)
    g = H.GpuLayer(qsa)
    ref = O.OracleLayer(O.QsaShape.of(wl), max_ctx=g.cfg.max_ctx)
    pre = synth.prefill_tokens(wl, 0, n0)
    g.append(pre["k"], pre["v"], pre["idx"])
    g.update()
    ref.append_tokens(pre["k"], pre["v"], pre["idx"])
    ref.update_pooled_cache()
    for step in range(6):
        st = synth.step_inputs(wl, 0, step)
        d = {k: H.to_dev(x) for k, x in st.items()}
        qsa.decode_step(0, d["k"], d["v"], d["idx"], d["q_idx"], d["w"], d["q"], g.outs["sel"], g.outs["n_sel"],
                        g.outs["out"])
        got = g.fetch()
        r = ref.decode_step(st["k"], st["v"], st["idx"], st["q_idx"], st["w"], st["q"])
        H.selection_mismatch(got["sel"], r["scores"], wl.k_blocks, H.CHAIN_GAP_REL)
        cells = O.expand_cells(got["sel"], ref.n)
        H.assert_attention_close(got["out"], O.sparse_attention(st["q"], ref.k, ref.v, cells, ref.shape))
    assert g.state() == (n0 + 6, (n0 + 6) // 4, 0)
    qsa.invalidate_pooled_cache(0, 5)
    g.index_topk(synth.step_inputs(wl, 0, 9)["q_idx"], synth.step_inputs(wl, 0, 9)["w"])
    assert len(g.fetch()["sel"]) == 0
    assert g.state(clear=True)[2] == 3  # QSA_ERR_STATE
