"""GPU parity of the multi-query verification step and of rollback.

Speculative decoding must not corrupt the cached pooled range ("Part 10", section
"incremental pooled-key cache（COMMON-004）"). A verification step appends T drafted
tokens and runs the index scan (one pass for all T queries), the selection and the
attention for every query at once; query u sees exactly what a single-token step at its
own token would. Rejected drafts are dropped with qsa_rollback, after which the blocks
they completed are pooled again from the accepted tokens.
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


def _drafts(wl, T, step0=0):
    """T consecutive single-token inputs stacked into [T, ...] arrays."""
    st = [synth.step_inputs(wl, 0, step0 + u) for u in range(T)]
    return {k: np.stack([s[k] for s in st]) for k in st[0]}


class Pair:
    """A GPU layer and an oracle layer fed the same tokens."""

    def __init__(self, wl_name, n0, max_extra=16, **cfg_kw):
        import sparse_attention_decode_02_b200 as Q
        self.wl = wl = synth.workload(wl_name)
        self.qsa = Q.Qsa(H.config_of(wl, max_ctx=((n0 + max_extra + 3) // 4) * 4, **cfg_kw))
        self.g = H.GpuLayer(self.qsa)
        self.ref = O.OracleLayer(O.QsaShape.of(wl), max_ctx=self.g.cfg.max_ctx)
        pre = synth.prefill_tokens(wl, 0, n0)
        self.g.append(pre["k"], pre["v"], pre["idx"])
        self.g.update()
        self.ref.append_tokens(pre["k"], pre["v"], pre["idx"])
        self.ref.update_pooled_cache()

    def gpu_multi(self, x):
        import sparse_attention_decode_02_b200 as Q
        T = len(x["k"])
        o = Q.alloc_multi_outputs(self.g.cfg, T)
        self.g.append(x["k"], x["v"], x["idx"])
        self.g.update()
        self.qsa.index_topk_multi(0, H.to_dev(x["q_idx"]), H.to_dev(x["w"].astype(np.float32)), o["sel"], o["n_sel"],
                                  o["scores"])
        self.qsa.sparse_attend_selected_multi(0, H.to_dev(x["q"]), o["sel"], o["n_sel"], o["out"])
        torch.cuda.synchronize()
        n_sel = o["n_sel"].cpu().numpy()
        return [{"sel": o["sel"][u, :n_sel[u]].cpu().numpy().astype(np.int64),
                 "scores": o["scores"][u].cpu().numpy().astype(np.float64),
                 "out": o["out"][u].cpu().numpy().astype(np.float64)} for u in range(T)]


def _check_query(p, got, ref, n_u, x, u):
    """Stage-isolated checks of query u: scores and selection against the oracle scoring
    the GPU's own pooled rows (identical inputs), attention over the GPU's own selection;
    plus the end-to-end selection against the oracle's own chain (its own pooled cache)."""
    b = n_u // 4
    gpu_pooled = p.g.pooled_rows(0, b)
    s_iso = O.block_scores(gpu_pooled, x["q_idx"][u], x["w"][u], n_u, p.ref.shape)
    if b:
        assert np.abs(got["scores"][:b] - s_iso).max() <= H.SCORE_REL * np.abs(s_iso).max()
    H.selection_mismatch(got["sel"], s_iso, p.wl.k_blocks, H.TIE_GAP_REL)
    assert len(ref["scores"]) == b
    H.selection_mismatch(got["sel"], ref["scores"], p.wl.k_blocks, H.CHAIN_GAP_REL)
    cells = O.expand_cells(got["sel"], n_u)
    H.assert_attention_close(got["out"], O.sparse_attention(x["q"][u], p.ref.k, p.ref.v, cells, p.ref.shape))


@pytest.mark.parametrize("wl_name,n0,T", [("tiny", 1016, 1), ("tiny", 1017, 2), ("tiny", 1018, 3),
                                          ("tiny", 1019, 4), ("tiny", 1020, 4), ("tiny", 1021, 3),
                                          ("ctx64k", 61789 - 4, 4), ("ctx64k", 61789 - 3, 2),
                                          ("ctx64k", 61789 - 2, 3)])   # 3 queries x 16 heads: MMA N = 96
def test_multi_query_step_matches_oracle(wl_name, n0, T):
    p = Pair(wl_name, n0)
    x = _drafts(p.wl, T)
    got = p.gpu_multi(x)
    ref = p.ref.multi_query_step(x["k"], x["v"], x["idx"], x["q_idx"], x["w"], x["q"])
    n = n0 + T
    assert p.g.state() == (n, n // 4, 0)
    H.assert_pooled_close(p.g.pooled_rows(0, n // 4), p.ref.pooled.rows[: n // 4])
    for u in range(T):
        _check_query(p, got[u], ref[u], n - T + u + 1, x, u)


def test_multi_query_equals_single_token_steps_on_gpu():
    """The fused T-query pass selects what T single-token steps select on the same caches."""
    wl = synth.workload("tiny")
    a, b = Pair("tiny", 1018), Pair("tiny", 1018)
    x = _drafts(wl, 4, step0=2)
    multi = a.gpu_multi(x)
    for u in range(4):
        single = b.g.step({k: x[k][u] for k in ("k", "v", "idx", "q_idx", "w", "q")})
        n_u = 1018 + u + 1
        s1 = single["scores"][: n_u // 4]
        np.testing.assert_allclose(multi[u]["scores"][: n_u // 4], s1, rtol=0, atol=1e-6 * np.abs(s1).max())
        if H.selection_mismatch(multi[u]["sel"], s1, wl.k_blocks, H.TIE_GAP_REL) == 0:
            np.testing.assert_allclose(multi[u]["out"], single["out"], rtol=0, atol=1e-5)
        # either way, each output matches the oracle attending over that query's own cells
        k_all = np.concatenate([a.ref.k[:1018], x["k"]])
        v_all = np.concatenate([a.ref.v[:1018], x["v"]])
        for res in (multi[u], single):
            H.assert_attention_close(res["out"], O.sparse_attention(x["q"][u], k_all, v_all,
                                                                    O.expand_cells(res["sel"], n_u), a.ref.shape))


def test_rollback_recomputes_dirty_blocks():
    """n0 = 4m+2: draft token n0+1 completes block m. Accept one draft, reject three; the
    next step (a different token at the rejected position) must match an oracle that never
    saw the rejected drafts, pooled block m included."""
    n0 = 4 * 253 + 2
    p = Pair("tiny", n0)
    wl = p.wl
    x = _drafts(wl, 4)
    p.gpu_multi(x)
    assert p.g.state() == (n0 + 4, (n0 + 4) // 4, 0)
    p.qsa.rollback(0, n0 + 1)
    assert p.g.state() == (n0 + 1, n0 // 4, 0)
    p.ref.multi_query_step(x["k"][:1], x["v"][:1], x["idx"][:1], x["q_idx"][:1], x["w"][:1], x["q"][:1])
    nxt = synth.step_inputs(wl, 0, 40)
    # fused decode append (pools block m again from the accepted tokens), then the step
    p.qsa.decode_append(0, H.to_dev(nxt["k"]), H.to_dev(nxt["v"]), H.to_dev(nxt["idx"]))
    p.g.index_topk(nxt["q_idx"], nxt["w"])
    p.g.gather()
    p.g.attend(nxt["q"])
    got = p.g.fetch()
    ref = p.ref.decode_step(nxt["k"], nxt["v"], nxt["idx"], nxt["q_idx"], nxt["w"], nxt["q"])
    n = n0 + 2
    assert p.g.state() == (n, n // 4, 0)
    H.assert_pooled_close(p.g.pooled_rows(0, n // 4), p.ref.pooled.rows[: n // 4])
    H.selection_mismatch(got["sel"], ref["scores"], wl.k_blocks, H.CHAIN_GAP_REL)
    H.assert_attention_close(got["out"], O.sparse_attention(nxt["q"], p.ref.k, p.ref.v, got["cells"], p.ref.shape))


def test_multi_query_limits_and_short_context():
    import sparse_attention_decode_02_b200 as Q
    p = Pair("tiny", 2, max_extra=8)
    x = _drafts(p.wl, 4)
    o = Q.alloc_multi_outputs(p.g.cfg, 4)
    for bad in (0, 5):
        q_idx = torch.zeros(max(bad, 1), p.wl.n_idx_heads, p.wl.d_idx, dtype=torch.float16, device="cuda")
        with pytest.raises(Q.QsaError) as e:
            st = p.qsa.lib.qsa_index_topk_multi(p.qsa.handle, 0, bad, q_idx.data_ptr(), o["scores"].data_ptr(),
                                                o["sel"].data_ptr(), o["n_sel"].data_ptr(), None, None)
            p.qsa._check(st)
        assert e.value.status == 1
    # 2 tokens in the cache but 4 queries: the first query would sit before token 0
    p.qsa.index_topk_multi(0, H.to_dev(x["q_idx"]), H.to_dev(x["w"].astype(np.float32)), o["sel"], o["n_sel"])
    torch.cuda.synchronize()
    assert p.g.state(clear=True)[2] == 3  # QSA_ERR_STATE
    assert o["n_sel"][0].item() == 0
    # rollback below zero is refused on the host; rollback past n_ctx changes nothing
    with pytest.raises(Q.QsaError):
        p.qsa.rollback(0, -1)
    p.qsa.rollback(0, 100)
    assert p.g.state()[:2] == (2, 0)


@pytest.mark.parametrize("T", [2, 4])
def test_multi_query_early_inputs_identical(T):
    """early_inputs (the scan builds the T-query operand before its dependency wait; here
    the append and pooled update right before it move the length, so the operand is
    rebuilt after the wait) against the default, bit for bit, over several draft rounds."""
    a = Pair("tiny", 4 * 250 + 1, max_extra=32, early_inputs=1)
    b = Pair("tiny", 4 * 250 + 1, max_extra=32)
    for r in range(4):
        x = _drafts(a.wl, T, step0=T * r)
        ga, gb = a.gpu_multi(x), b.gpu_multi(x)
        for u in range(T):
            np.testing.assert_array_equal(ga[u]["sel"], gb[u]["sel"])
            np.testing.assert_array_equal(ga[u]["scores"], gb[u]["scores"])
            np.testing.assert_array_equal(ga[u]["out"], gb[u]["out"])
