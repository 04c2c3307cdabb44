"""GPU parity of the context-parallel decode step, with the shards emulated on one GPU.

A layer's context is split into contiguous, block-aligned shards (the last one holds the
open tail); each shard is its own library context, pooled at its blocks' global positions
(rope_pos_offset = 4 * first block). One step: every shard's local top-K as candidate
slots (qsa_cp_index_candidates), the global top-K of all slots (qsa_cp_select), every
shard's attention partial over its part of it (qsa_cp_attend_partial) and the exact
merge (qsa_cp_merge). The exchange between devices is replaced by stacking the slots and
partials in one process. The selection must equal the single-device selection bit for
bit (the shards compute the same scores), every shard's candidates and partials must
match the oracle's sharded form, and the merged output must match the oracle's attention
over the single-device cells ("Part 10", section "QSAとQSA indexerについて": long context by
sparsity; the sharded form is exact).
"""
import numpy as np
import pytest
import torch

import synth
from oracle import qsa_oracle as O
from tests import gpu_harness as H

pytestmark = pytest.mark.gpu

LSE_ABS = 2e-3  # log-sum-exp of f32 logits against float64 (the attention's den to ~1e-3 relative)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    H.ensure_library()


def _bounds(n, shards):
    starts = [4 * ((r * (n // 4)) // shards) for r in range(shards)]
    return starts + [n]


def _shard(wl, pre, t0, t1, top_k_tokens):
    import sparse_attention_decode_02_b200 as Q
    cfg = H.config_of(wl, max_ctx=(t1 - t0 + 7) // 4 * 4, top_k_tokens=top_k_tokens, rope_pos_offset=t0)
    qsa = Q.Qsa(cfg)
    g = H.GpuLayer(qsa)
    g.append(pre["k"][t0:t1], pre["v"][t0:t1], pre["idx"][t0:t1])
    g.update()
    return qsa, g


CASES = [("tiny", 1027, 2, None), ("tiny", 1027, 3, None), ("tiny", 1026, 4, None), ("tiny", 1027, 3, 1024),
         ("ctx64k", 61790, 2, None), ("ctx64k", 61790, 4, None)]


@pytest.mark.parametrize("wl_name,n,shards,topk", CASES,
                         ids=[f"{c[0]}-n{c[1]}-x{c[2]}-k{c[3] or 'def'}" for c in CASES])
def test_context_parallel_step_equals_single_device(wl_name, n, shards, topk):
    import sparse_attention_decode_02_b200 as Q
    wl = synth.workload(wl_name)
    top_k_tokens = topk or wl.top_k_tokens
    shape = O.QsaShape.of(wl)
    if topk:
        shape = O.QsaShape(shape.d_idx, shape.n_idx_heads, topk, shape.n_q_heads, shape.n_kv_heads, shape.head_dim,
                           shape.rope_base, shape.rms_eps)
    K = top_k_tokens // 4
    pre = synth.prefill_tokens(wl, 0, n)
    st = synth.step_inputs(wl, 0, 0)
    d = {k: H.to_dev(x) for k, x in st.items()}
    bounds = _bounds(n, shards)

    # ---- the single-device step on the whole context ----
    one = Q.Qsa(H.config_of(wl, max_ctx=(n + 7) // 4 * 4, top_k_tokens=top_k_tokens))
    g1 = H.GpuLayer(one)
    g1.append(pre["k"], pre["v"], pre["idx"])
    g1.update()
    g1.index_topk(st["q_idx"], st["w"])
    g1.attend_selected(st["q"])
    single = g1.fetch()

    # ---- the sharded step ----
    cand_s = torch.empty(shards, K, dtype=torch.float32, device="cuda")
    cand_b = torch.empty(shards, K, dtype=torch.int32, device="cuda")
    n_cand = torch.empty(shards, dtype=torch.int32, device="cuda")
    layers = []
    for r in range(shards):
        t0, t1 = bounds[r], bounds[r + 1]
        qsa, g = _shard(wl, pre, t0, t1, top_k_tokens)
        qsa.cp_index_candidates(0, d["q_idx"], d["w"], n, t0 // 4, cand_s[r], cand_b[r], n_cand[r:r + 1])
        layers.append((qsa, g, t0, t1))
    sel = torch.empty(K, dtype=torch.int32, device="cuda")
    n_sel = torch.empty(1, dtype=torch.int32, device="cuda")
    Q.cp_select(cand_s, cand_b, shards, K, sel, n_sel)
    o_parts = torch.empty(shards, wl.n_q_heads, wl.head_dim, dtype=torch.float32, device="cuda")
    lse_parts = torch.empty(shards, wl.n_q_heads, dtype=torch.float32, device="cuda")
    for r, (qsa, g, t0, t1) in enumerate(layers):
        qsa.cp_attend_partial(0, d["q"], sel, n_sel, t0 // 4, o_parts[r], lse_parts[r])
    out = torch.empty(wl.n_q_heads, wl.head_dim, dtype=torch.float32, device="cuda")
    Q.cp_merge(o_parts, lse_parts, shards, wl.n_q_heads, wl.head_dim, out)
    torch.cuda.synchronize()

    # the selection: the single device's, bit for bit
    ns = int(n_sel[0])
    got_sel = sel[:ns].cpu().numpy().astype(np.int64)
    np.testing.assert_array_equal(got_sel, single["sel"])
    # every shard's candidates against the oracle's sharded form (the oracle's own pooling
    # of the shard's raw keys at their global positions)
    for r, (qsa, g, t0, t1) in enumerate(layers):
        b0, b1 = t0 // 4, t1 // 4
        mine = O.pooled_summaries(pre["idx"], b0, b1, shape)
        s_ref, b_ref = O.shard_candidates(mine, b0, st["q_idx"], st["w"], n, shape)
        nc = int(n_cand[r])
        assert nc == len(b_ref)
        cb = cand_b[r].cpu().numpy().astype(np.int64)
        cs = cand_s[r].cpu().numpy().astype(np.float64)
        assert np.all(cb[nc:] == -1) and np.all(np.isneginf(cs[nc:]))
        # the shard's pooled rows (global positions) against the oracle's; its scores
        # against the oracle scoring the shard's own f16 rows (identical inputs)
        gp = g.pooled_rows(0, b1 - b0)
        H.assert_pooled_close(gp, mine)
        all_scores = O.block_scores(gp, st["q_idx"], st["w"], n, shape) if b1 > b0 else np.zeros(0)
        H.selection_mismatch(cb[:nc] - b0, all_scores, K, H.TIE_GAP_REL)
        H.selection_mismatch(cb[:nc] - b0, O.block_scores(mine, st["q_idx"], st["w"], n, shape), K,
                             H.CHAIN_GAP_REL)
        if nc:
            assert np.abs(cs[:nc] - all_scores[cb[:nc] - b0]).max() <= H.SCORE_REL * np.abs(all_scores).max()
        # the partial over this shard's part of the selection, against the oracle's
        mine_sel = got_sel[(got_sel >= b0) & (got_sel < b1)]
        cells = O.expand_cells(mine_sel, t1)
        cells = cells[cells >= t0]
        o_ref, lse_ref = O.attention_partial(st["q"], pre["k"], pre["v"], cells, shape)
        lse_got = lse_parts[r].cpu().numpy().astype(np.float64)
        if len(cells):
            H.assert_attention_close(o_parts[r].cpu().numpy().astype(np.float64), o_ref)
            assert np.abs(lse_got - lse_ref).max() <= LSE_ABS
        else:
            assert np.all(np.isneginf(lse_got)) and not o_parts[r].cpu().numpy().any()
    # the merged output against the oracle over the single-device cells
    ref_out = O.sparse_attention(st["q"], pre["k"], pre["v"], O.expand_cells(single["sel"], n), shape)
    H.assert_attention_close(out.cpu().numpy().astype(np.float64), ref_out)
    H.assert_attention_close(out.cpu().numpy().astype(np.float64), single["out"])
    for qsa, g, _, _ in layers:
        assert g.state()[2] == 0


def test_context_parallel_empty_shard_and_select_limits():
    """A shard none of whose blocks is selected (and without the tail) gives out = 0 and
    lse = -inf, and the merge ignores it; qsa_cp_select refuses more than 8192 slots."""
    import sparse_attention_decode_02_b200 as Q
    wl = synth.workload("tiny")
    n = 1024
    pre = synth.prefill_tokens(wl, 0, n)
    st = synth.step_inputs(wl, 0, 1)
    qsa, g = _shard(wl, pre, 0, 512, wl.top_k_tokens)
    sel = torch.tensor([200, 201, 250], dtype=torch.int32, device="cuda")   # blocks of another shard
    n_sel = torch.tensor([3], dtype=torch.int32, device="cuda")
    o = torch.full((wl.n_q_heads, wl.head_dim), float("nan"), device="cuda")
    lse = torch.zeros(wl.n_q_heads, device="cuda")
    qsa.cp_attend_partial(0, H.to_dev(st["q"]), sel, n_sel, 0, o, lse)
    torch.cuda.synchronize()
    assert not o.cpu().numpy().any() and np.all(np.isneginf(lse.cpu().numpy()))
    # merged with a non-empty partial: that partial unchanged
    o2 = torch.randn(wl.n_q_heads, wl.head_dim, device="cuda")
    lse2 = torch.randn(wl.n_q_heads, device="cuda")
    out = torch.empty_like(o2)
    Q.cp_merge(torch.stack([o, o2]), torch.stack([lse, lse2]), 2, wl.n_q_heads, wl.head_dim, out)
    torch.cuda.synchronize()
    torch.testing.assert_close(out, o2, rtol=1e-6, atol=1e-6)
    big = torch.zeros(9, 1024, device="cuda")
    with pytest.raises(Q.QsaError) as err:
        Q.cp_select(big, big.to(torch.int32), 9, 1024, sel, n_sel)
    assert err.value.status == 5  # QSA_ERR_UNSUPPORTED
