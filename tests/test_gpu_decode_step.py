"""GPU parity of qsa_decode_step, the whole per-layer step in one call.

When the pooled cache is current up to the previous token, the call runs three launches:
the indexer-scan kernel itself appends the token and pools the block the token completes
("Part 10", section "incremental pooled-key cache（COMMON-004）": only the new block is
computed), then the selection (starting from the scan's score-key histogram), then the
attention. These tests hold it bit for bit to the separate calls (qsa_decode_append,
qsa_index_topk, qsa_sparse_attend_selected) over several block completions, for the
default layer, the RoPE switches and the FP8 K/V cache, check it against the oracle
(adversarial tables for the histogram-started selection included), and cover the form
taken after a bulk append and the capacity limit.
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


def _layer(wl, n0, extra=16, **cfg_kw):
    import sparse_attention_decode_02_b200 as Q
    qsa = Q.Qsa(H.config_of(wl, max_ctx=(n0 + extra + 3) // 4 * 4, **cfg_kw))
    g = H.GpuLayer(qsa)
    pre = synth.prefill_tokens(wl, 0, n0)
    g.append(pre["k"], pre["v"], pre["idx"])
    return qsa, g, pre


def _decode_step(qsa, g, st):
    d = {k: H.to_dev(x) for k, x in st.items()}
    qsa.decode_step(0, d["k"], d["v"], d["idx"], d["q_idx"], d["w"], d["q"], g.outs["sel"], g.outs["n_sel"],
                    g.outs["out"])


def _separate(qsa, g, st):
    qsa.decode_append(0, H.to_dev(st["k"]), H.to_dev(st["v"]), H.to_dev(st["idx"]))
    g.index_topk(st["q_idx"], st["w"])
    g.attend_selected(st["q"])


VARIANTS = [
    ("tiny", {}),
    ("tiny", dict(rope_interleaved=True)),
    ("tiny", dict(rope_dims=32, rope_pos_stride=1, rope_pos_offset=3)),
    ("tiny", dict(kv_format=1)),
    ("ctx64k", {}),
]


@pytest.mark.parametrize("wl_name,kw", VARIANTS, ids=[f"{w}-{'-'.join(map(str, k.items())) or 'default'}"
                                                      for w, k in VARIANTS])
def test_decode_step_equals_separate_calls_over_block_completions(wl_name, kw):
    wl = synth.workload(wl_name)
    n0 = 1017 if wl_name == "tiny" else 8193
    qa, ga, _ = _layer(wl, n0, **kw)
    qb, gb, _ = _layer(wl, n0, **kw)
    ga.update()
    gb.update()
    for step in range(11):  # n = n0 + 1 .. n0 + 11: three block completions
        st = synth.step_inputs(wl, 0, step)
        _decode_step(qa, ga, st)
        _separate(qb, gb, st)
        torch.cuda.synchronize()
        na, nb = int(ga.outs["n_sel"][0]), int(gb.outs["n_sel"][0])
        assert na == nb == min(wl.k_blocks, (n0 + step + 1) // 4)
        assert torch.equal(ga.outs["sel"][:na], gb.outs["sel"][:nb]), f"step {step}: selection"
        assert torch.equal(ga.outs["out"], gb.outs["out"]), f"step {step}: attention output"
        assert ga.state() == gb.state() == (n0 + step + 1, (n0 + step + 1) // 4, 0)
    n = n0 + 11
    for key in ("k_cache", "v_cache", "idx_cache", "pooled_cache") + (("kv_scales",) if kw.get("kv_format") else ()):
        assert torch.equal(ga.buf[key], gb.buf[key]), key
    # the live pooled cache equals a full rebuild
    live = ga.pooled_rows(0, n // 4)
    qa.invalidate_pooled_cache(0, 0)
    ga.buf["pooled_cache"].zero_()
    ga.update()
    np.testing.assert_array_equal(ga.pooled_rows(0, n // 4), live)


def test_decode_step_matches_oracle_every_step():
    """The fused step against the oracle's own chain: pooled rows, selection (near-tie
    flips only), attention over the GPU's cells."""
    wl = synth.workload("tiny")
    n0 = 1017
    qsa, g, pre = _layer(wl, n0)
    g.update()
    ref = O.OracleLayer(O.QsaShape.of(wl), max_ctx=g.cfg.max_ctx)
    ref.append_tokens(pre["k"], pre["v"], pre["idx"])
    ref.update_pooled_cache()
    for step in range(9):
        st = synth.step_inputs(wl, 0, step)
        _decode_step(qsa, g, st)
        got = g.fetch()
        r = ref.decode_step(st["k"], st["v"], st["idx"], st["q_idx"], st["w"], st["q"])
        n = ref.n
        H.assert_pooled_close(g.pooled_rows(0, n // 4), ref.pooled.rows[: n // 4])
        flips = H.selection_mismatch(got["sel"], r["scores"], wl.k_blocks, H.CHAIN_GAP_REL)
        H.record_chain("tiny-decode-step", step, flips)
        cells = O.expand_cells(got["sel"], n)
        want = r["out"] if np.array_equal(cells, r["cells"]) else O.sparse_attention(st["q"], ref.k, ref.v, cells,
                                                                                     ref.shape)
        H.assert_attention_close(got["out"], want)
    assert g.state() == (n0 + 9, (n0 + 9) // 4, 0)


def test_decode_step_after_bulk_append_pools_waiting_blocks():
    """After qsa_append_tokens without a pooled update, the step pools every waiting block
    first (the four-launch form), then continues in the three-launch form."""
    wl = synth.workload("tiny")
    n0 = 1019
    qa, ga, pre = _layer(wl, n0)           # no update: 254 blocks waiting
    qb, gb, _ = _layer(wl, n0)
    gb.update()
    for step in range(6):
        st = synth.step_inputs(wl, 0, step)
        _decode_step(qa, ga, st)
        _separate(qb, gb, st)
        torch.cuda.synchronize()
        assert ga.state() == gb.state() == (n0 + step + 1, (n0 + step + 1) // 4, 0)
        assert torch.equal(ga.outs["out"], gb.outs["out"])
    n = n0 + 6
    np.testing.assert_array_equal(ga.pooled_rows(0, n // 4), gb.pooled_rows(0, n // 4))


def test_decode_step_reports_capacity_and_writes_nothing():
    wl = synth.workload("tiny")
    n0 = 1022
    qsa, g, pre = _layer(wl, n0, extra=0)   # max_ctx = 1024: two more tokens fit
    g.update()
    for step in range(2):
        _decode_step(qsa, g, synth.step_inputs(wl, 0, step))
    assert g.state() == (1024, 256, 0)
    before = {k: g.buf[k].clone() for k in ("k_cache", "v_cache", "idx_cache", "pooled_cache")}
    _decode_step(qsa, g, synth.step_inputs(wl, 0, 2))
    n, p, status = g.state(clear=True)
    assert (n, p) == (1024, 256) and status == 2  # QSA_ERR_CAPACITY
    for k, t in before.items():
        assert torch.equal(g.buf[k], t), k


@pytest.mark.parametrize("table", ["repeats10", "allequal", "zeroquery", "random"])
@pytest.mark.parametrize("wl_name,n0", [("tiny", 4 * 600 + 1), ("ctx256k_12l", 255181)])
def test_decode_step_selection_on_adversarial_tables(wl_name, n0, table):
    """The decode step's selection (started from the scan's score-key histogram) on pooled
    tables that take every path of the radix passes: exact ties within and across CTAs
    (rows repeating ten base rows, one row everywhere, a zero query so that every score is
    0 and the whole key decides by block order) and plain N(0,1) rows. The selection must
    be the oracle's on the same f16 table (ties to the lower block)."""
    wl = synth.workload(wl_name)
    qsa, g, pre = _layer(wl, n0, extra=8)
    g.update()
    B = n0 // 4
    base = synth.random_pooled(wl, 0, 10, salt=3)
    if table == "repeats10":
        pooled = base[np.arange(B) % 10]
    elif table == "allequal":
        pooled = np.repeat(base[:1], B, axis=0)
    else:
        pooled = synth.random_pooled(wl, 0, B, salt=11)
    g.buf["pooled_cache"][:B] = H.to_dev(pooled)
    st = dict(synth.step_inputs(wl, 0, 0))   # n0 + 1 tokens: no block completes
    if table == "zeroquery":
        st["q_idx"] = np.zeros_like(st["q_idx"])
    _decode_step(qsa, g, st)
    torch.cuda.synchronize()
    n = n0 + 1
    assert n % 4 != 0 and g.state() == (n, B, 0)
    got = g.outs["sel"][: int(g.outs["n_sel"][0])].cpu().numpy().astype(np.int64)
    ref_scores = O.block_scores(pooled, st["q_idx"], st["w"], n, O.QsaShape.of(wl))
    gap = 0.0 if table in ("repeats10", "allequal", "zeroquery") else H.TIE_GAP_REL
    H.selection_mismatch(got, ref_scores, wl.k_blocks, gap)
    if table in ("allequal", "zeroquery"):
        assert got.tolist() == list(range(wl.k_blocks))


@pytest.mark.parametrize("wl_name,kw", [("tiny", {}), ("tiny", dict(rope_dims=32, rope_pos_stride=1)),
                                        ("ctx64k", {}), ("ctx64k", dict(pooled_format=1))],
                         ids=["tiny", "tiny-partial-rope", "ctx64k", "ctx64k-fp8-pooled"])
def test_early_inputs_give_identical_results(wl_name, kw):
    """early_inputs = QSA_INPUTS_EARLY (the scan prepares the query before waiting for the
    previous kernel) against the default, bit for bit: the decode step over block
    completions, and the separate calls, where the append that precedes the scan changes
    the length after the scan read it early (the scan then rebuilds the query operand)."""
    wl = synth.workload(wl_name)
    n0 = 1017 if wl_name == "tiny" else 8193
    qa, ga, _ = _layer(wl, n0, extra=24, early_inputs=1, **kw)
    qb, gb, _ = _layer(wl, n0, extra=24, **kw)
    ga.update()
    gb.update()
    for step in range(12):
        st = synth.step_inputs(wl, 0, step)
        if step % 2 == 0:
            _decode_step(qa, ga, st)
            _decode_step(qb, gb, st)
        else:
            _separate(qa, ga, st)
            _separate(qb, gb, st)
        torch.cuda.synchronize()
        na, nb = int(ga.outs["n_sel"][0]), int(gb.outs["n_sel"][0])
        assert na == nb
        assert torch.equal(ga.outs["sel"][:na], gb.outs["sel"][:nb]), f"step {step}: selection"
        assert torch.equal(ga.outs["out"], gb.outs["out"]), f"step {step}: attention output"
        if step % 2:
            assert torch.equal(ga.scores, gb.scores), f"step {step}: scores"
        assert ga.state() == gb.state() == (n0 + step + 1, (n0 + step + 1) // 4, 0)


def _layers(wl, n0, n_layers, extra=16, **cfg_kw):
    import sparse_attention_decode_02_b200 as Q
    qsa = Q.Qsa(H.config_of(wl, max_ctx=(n0 + extra + 3) // 4 * 4, n_layers=n_layers, **cfg_kw))
    gs = []
    for layer in range(n_layers):
        g = H.GpuLayer(qsa, layer)
        pre = synth.prefill_tokens(wl, layer, n0)
        g.append(pre["k"], pre["v"], pre["idx"])
        g.update()
        gs.append(g)
    return qsa, gs


def _decode_step_layer(qsa, g, st):
    d = {k: H.to_dev(x) for k, x in st.items()}
    qsa.decode_step(g.layer, d["k"], d["v"], d["idx"], d["q_idx"], d["w"], d["q"], g.outs["sel"],
                    g.outs["n_sel"], g.outs["out"])


def test_back_to_back_layers_equal_synchronised_steps():
    """Steps of three layers enqueued back to back (each layer's kernels launching while
    the previous layer's still run, and preparing their inputs and prefetches before their
    dependency waits) equal the same steps with a synchronisation after every call, bit
    for bit, over block completions."""
    wl = synth.workload("ctx64k")
    n0, L = 8190, 3
    qa, ga = _layers(wl, n0, L, early_inputs=1)
    qb, gb = _layers(wl, n0, L, early_inputs=1)
    for step in range(7):
        sts = [synth.step_inputs(wl, layer, step) for layer in range(L)]
        ins = [{k: H.to_dev(x) for k, x in st.items()} for st in sts]  # copied before the steps
        torch.cuda.synchronize()
        for layer in range(L):
            d = ins[layer]
            qa.decode_step(layer, d["k"], d["v"], d["idx"], d["q_idx"], d["w"], d["q"], ga[layer].outs["sel"],
                           ga[layer].outs["n_sel"], ga[layer].outs["out"])
        torch.cuda.synchronize()
        for layer in range(L):
            _decode_step_layer(qb, gb[layer], sts[layer])
            torch.cuda.synchronize()
        for layer in range(L):
            a, b = ga[layer].outs, gb[layer].outs
            na, nb = int(a["n_sel"][0]), int(b["n_sel"][0])
            assert na == nb == wl.k_blocks
            assert torch.equal(a["sel"][:na], b["sel"][:nb]), f"step {step} layer {layer}: selection"
            assert torch.equal(a["out"], b["out"]), f"step {step} layer {layer}: attention output"
            assert ga[layer].state() == gb[layer].state() == (n0 + step + 1, (n0 + step + 1) // 4, 0)


def test_pooled_rewrite_right_before_a_step_is_seen():
    """A pooled update enqueued right before a decode step (no synchronisation) rewrites
    rows that the step's scan reads: the scan sees the rewritten rows, not the ones before.
    The rows are first overwritten with a large value, so a read of them before the update
    completed would change the selection."""
    wl = synth.workload("ctx64k")
    n0 = 8193
    qa, ga, _ = _layer(wl, n0, extra=24, early_inputs=1)
    qb, gb, _ = _layer(wl, n0, extra=24, early_inputs=1)
    ga.update()
    gb.update()
    for step in range(3):
        st = synth.step_inputs(wl, 0, step)
        _decode_step(qa, ga, st)
        _decode_step(qb, gb, st)
    torch.cuda.synchronize()
    n = n0 + 3
    ga.buf["pooled_cache"].view(torch.int16)[: n // 4].fill_(0x7BFF)  # f16 65504
    qa.invalidate_pooled_cache(0, 0)
    ga.update()
    st = synth.step_inputs(wl, 0, 3)
    _decode_step(qa, ga, st)  # enqueued right behind the update
    _decode_step(qb, gb, st)
    torch.cuda.synchronize()
    na, nb = int(ga.outs["n_sel"][0]), int(gb.outs["n_sel"][0])
    assert na == nb
    assert torch.equal(ga.outs["sel"][:na], gb.outs["sel"][:nb])
    assert torch.equal(ga.outs["out"], gb.outs["out"])
    np.testing.assert_array_equal(ga.pooled_rows(0, (n + 1) // 4), gb.pooled_rows(0, (n + 1) // 4))
