"""GPU parity of the CUDA path (through the C ABI) against the CPU oracle.

Stage-isolated checks feed both sides identical inputs drawn by `synth` (or computed by
the oracle): pooled cache from raw keys, scores + selection from one f16 pooled table,
attention from one cell list. End-to-end chains let each side compute everything.
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


def _qsa(wl, **kw):
    import sparse_attention_decode_02_b200 as Q
    return Q.Qsa(H.config_of(wl, **kw))


def _prefilled(wl, n=None, layer=0, **kw):
    """A GPU layer and an oracle layer holding the same prefill."""
    qsa = _qsa(wl, **kw)
    g = H.GpuLayer(qsa)
    shape = O.QsaShape.of(wl)
    if "top_k_tokens" in kw:
        shape = O.QsaShape(shape.d_idx, shape.n_idx_heads, kw["top_k_tokens"], shape.n_q_heads,
                           shape.n_kv_heads, shape.head_dim, shape.rope_base, shape.rms_eps)
    ref = O.OracleLayer(shape, max_ctx=g.cfg.max_ctx)
    pre = synth.prefill_tokens(wl, layer, n)
    if len(pre["k"]):
        g.append(pre["k"], pre["v"], pre["idx"])
        g.update()
        ref.append_tokens(pre["k"], pre["v"], pre["idx"])
        ref.update_pooled_cache()
    return qsa, g, ref


def _ref_attention_over(gpu_cells, r, st, ref, wl):
    """The oracle's attention output for the cells the GPU attended: the oracle's own output
    when the cell lists agree, else the oracle attending over the GPU's cells."""
    if np.array_equal(gpu_cells, r["cells"]):
        return r["out"]
    return O.sparse_attention(st["q"], ref.k, ref.v, np.asarray(gpu_cells, np.int64), O.QsaShape.of(wl))


# ----------------------------------------------------------------------------- pooled cache

def test_pooled_cache_matches_oracle_and_full_rebuild():
    wl = synth.workload("tiny")
    qsa, g, ref = _prefilled(wl, n=1023)
    n = 1023
    for step in range(9):  # crosses two block boundaries
        st = synth.step_inputs(wl, 0, step)
        g.append(st["k"], st["v"], st["idx"])
        g.update()
        ref.append_tokens(st["k"][None], st["v"][None], st["idx"][None])
        ref.update_pooled_cache()
        n += 1
        assert g.state() == (n, n // 4, 0)
    inc = g.pooled_rows(0, n // 4)
    H.assert_pooled_close(inc, ref.pooled.rows[: n // 4])
    # incremental == full GPU recompute, bit for bit
    qsa.invalidate_pooled_cache(0, 0)
    g.buf["pooled_cache"].zero_()
    g.update()
    assert g.state() == (n, n // 4, 0)
    np.testing.assert_array_equal(g.pooled_rows(0, n // 4), inc)


def test_pooled_cache_with_gain_and_partial_invalidation():
    wl = synth.workload("tiny")
    gain = np.random.default_rng(3).random(wl.d_idx).astype(np.float32) + 0.5
    qsa = _qsa(wl)
    g = H.GpuLayer(qsa, gain=gain)
    pre = synth.prefill_tokens(wl, 0, 401)
    g.append(pre["k"], pre["v"], pre["idx"])
    g.update()
    full = O.pooled_cache_full(pre["idx"], 401, O.QsaShape.of(wl), gain=gain.astype(np.float64))
    H.assert_pooled_close(g.pooled_rows(0, 100), full)
    before = g.pooled_rows(0, 100)
    qsa.invalidate_pooled_cache(0, 37)
    assert g.state()[1] == 37
    g.buf["pooled_cache"][37:].zero_()
    g.update()
    np.testing.assert_array_equal(g.pooled_rows(0, 100), before)


# ----------------------------------------------------------------------------- selection

def _load_pooled(g, qsa, pooled, n):
    g.buf["pooled_cache"][: len(pooled)] = H.to_dev(pooled)
    qsa.restore_layer(0, n, n // 4)


@pytest.mark.parametrize("wl_name,n", [("tiny", 1027), ("tiny", 4 * 64 + 1), ("ctx64k", 4000 * 4 + 3),
                                       ("ctx64k", 61790), ("ctx256k_12l", 255182)])
def test_selection_stage_isolated(wl_name, n):
    wl = synth.workload(wl_name)
    qsa = _qsa(wl, max_ctx=((n + 3) // 4) * 4 + 4)
    g = H.GpuLayer(qsa)
    shape = O.QsaShape.of(wl)
    pooled = synth.random_pooled(wl, 0, n // 4, salt=n)
    _load_pooled(g, qsa, pooled, n)
    st = synth.step_inputs(wl, 0, 0)
    g.index_topk(st["q_idx"], st["w"])
    res = g.fetch()
    ref_scores = O.block_scores(pooled, st["q_idx"], st["w"], n, shape)
    gs = res["scores"][: n // 4]
    assert np.abs(gs - ref_scores).max() <= H.SCORE_REL * np.abs(ref_scores).max()
    mism = H.selection_mismatch(res["sel"], ref_scores, shape.k_blocks, H.TIE_GAP_REL)
    print(f"{wl_name} n={n}: selection mismatches within tie gap: {mism}")
    assert g.state()[2] == 0


def test_selection_exact_ties_take_lower_index():
    wl = synth.workload("tiny")
    n = 4 * 300 + 2
    qsa = _qsa(wl, max_ctx=n + 2)
    g = H.GpuLayer(qsa)
    base = synth.random_pooled(wl, 0, 10, salt=7)
    # every row repeats one of 10 rows: each score value occurs ~30 times
    pooled = base[np.arange(n // 4) % 10]
    _load_pooled(g, qsa, pooled, n)
    st = synth.step_inputs(wl, 0, 1)
    g.index_topk(st["q_idx"], st["w"])
    res = g.fetch()
    ref_scores = O.block_scores(pooled, st["q_idx"], st["w"], n, O.QsaShape.of(wl))
    # identical rows give bit-identical GPU scores, so the tie-break is exercised exactly
    assert H.selection_mismatch(res["sel"], ref_scores, wl.k_blocks, 0.0) == 0
    # all-equal scores: the first K blocks
    _load_pooled(g, qsa, np.repeat(base[:1], n // 4, axis=0), n)
    g.index_topk(st["q_idx"], st["w"])
    assert g.fetch()["sel"].tolist() == list(range(wl.k_blocks))


def test_selection_when_blocks_fit_in_k_and_stale_cache():
    wl = synth.workload("tiny")
    qsa, g, ref = _prefilled(wl, n=4 * 40 + 3)
    st = synth.step_inputs(wl, 0, 0)
    g.index_topk(st["q_idx"], st["w"])
    assert g.fetch()["sel"].tolist() == list(range(40))
    # append a full block without updating the pooled cache: the scan must refuse
    pre = synth.prefill_tokens(wl, 0, 4, first=163)
    g.append(pre["k"], pre["v"], pre["idx"])
    g.index_topk(st["q_idx"], st["w"])
    res = g.fetch()
    assert len(res["sel"]) == 0
    n, n_pooled, status = g.state(clear=True)
    assert (n, n_pooled, status) == (167, 40, 3)
    assert g.state()[2] == 0


# ----------------------------------------------------------------------------- attention

@pytest.mark.parametrize("wl_name,n_cells", [("tiny", 1), ("tiny", 7), ("tiny", 259), ("ctx64k", 2051),
                                              ("ctx64k", 600), ("ctx64k", 2048)])
def test_attention_stage_isolated(wl_name, n_cells):
    wl = synth.workload(wl_name)
    n = 4096 + 3
    qsa = _qsa(wl, max_ctx=n + 1)
    g = H.GpuLayer(qsa)
    pre = synth.prefill_tokens(wl, 0, n)
    g.append(pre["k"], pre["v"], pre["idx"])
    cells = synth.random_cells(wl, 0, n, n_cells, salt=n_cells)
    q = synth.step_inputs(wl, 0, 2)["q"]
    cells_d = torch.zeros(wl.max_cells, dtype=torch.int32, device="cuda")
    cells_d[: len(cells)] = H.to_dev(cells)
    nc = torch.tensor([len(cells)], dtype=torch.int32, device="cuda")
    g.attend(q, cells_d, nc)
    out = g.fetch()["out"]
    ref = O.sparse_attention(q, pre["k"], pre["v"], cells, O.QsaShape.of(wl))
    H.assert_attention_close(out, ref)


def test_full_selection_equals_dense_attention():
    """top-k covering every block == dense attention over all n tokens (torch float64 SDPA)."""
    wl = synth.workload("tiny")
    n0 = 4 * 64 - 3       # all blocks fit in the top-k
    qsa, g, ref = _prefilled(wl, n=n0)
    st = synth.step_inputs(wl, 0, 0)
    res = g.step(st)
    n = n0 + 1
    assert res["cells"].tolist() == list(range(n))
    pre = synth.prefill_tokens(wl, 0, n0)
    k_all = torch.from_numpy(np.concatenate([pre["k"], st["k"][None]]).astype(np.float64))
    v_all = torch.from_numpy(np.concatenate([pre["v"], st["v"][None]]).astype(np.float64))
    q = torch.from_numpy(st["q"].astype(np.float64)).reshape(1, wl.n_q_heads, 1, wl.head_dim)
    dense = torch.nn.functional.scaled_dot_product_attention(
        q, k_all.permute(1, 0, 2)[None], v_all.permute(1, 0, 2)[None], enable_gqa=True)
    H.assert_attention_close(res["out"], dense.reshape(wl.n_q_heads, wl.head_dim).numpy())


def test_empty_and_invalid_cells():
    wl = synth.workload("tiny")
    qsa, g, ref = _prefilled(wl, n=100)
    q = synth.step_inputs(wl, 0, 0)["q"]
    cells = torch.tensor([5, 7, 150, -2] + [0] * (wl.max_cells - 4), dtype=torch.int32, device="cuda")
    g.attend(q, cells, torch.tensor([0], dtype=torch.int32, device="cuda"))
    assert np.all(g.fetch()["out"] == 0)
    assert g.state()[2] == 0
    g.attend(q, cells, torch.tensor([4], dtype=torch.int32, device="cuda"))
    out = g.fetch()["out"]
    pre = synth.prefill_tokens(wl, 0, 100)
    H.assert_attention_close(out, O.sparse_attention(q, pre["k"], pre["v"], np.array([5, 7]), O.QsaShape.of(wl)))
    assert g.state(clear=True)[2] == 6


# ----------------------------------------------------------------------------- chains

def test_tiny_chain_matches_oracle_every_step():
    wl = synth.workload("tiny")
    qsa, g, ref = _prefilled(wl)
    flips = 0
    for step in range(wl.n_steps):
        st = synth.step_inputs(wl, 0, step)
        res = g.step(st)
        r = ref.decode_step(st["k"], st["v"], st["idx"], st["q_idx"], st["w"], st["q"])
        n = wl.n_prefill + step + 1
        H.assert_pooled_close(g.pooled_rows(0, n // 4), ref.pooled.rows[: n // 4])
        f = H.selection_mismatch(res["sel"], r["scores"], wl.k_blocks, H.CHAIN_GAP_REL)
        flips += f
        assert len(res["cells"]) == len(r["cells"])
        # attention is always checked: against the oracle's own output when the cells agree,
        # else against the oracle attending over the GPU's cells
        H.assert_attention_close(res["out"], _ref_attention_over(res["cells"], r, st, ref, wl))
        H.record_chain("tiny", step, f)
    print(f"tiny chain: {flips} near-tie selection flips over {wl.n_steps} steps")
    assert g.state() == (wl.n_prefill + wl.n_steps, (wl.n_prefill + wl.n_steps) // 4, 0)


def test_short_contexts_tail_only():
    wl = synth.workload("tiny")
    qsa = _qsa(wl)
    g = H.GpuLayer(qsa)
    ref = O.OracleLayer(O.QsaShape.of(wl), max_ctx=g.cfg.max_ctx)
    for step in range(6):  # n = 1..6: tail only, then one block
        st = synth.step_inputs(wl, 0, step)
        res = g.step(st)
        r = ref.decode_step(st["k"], st["v"], st["idx"], st["q_idx"], st["w"], st["q"])
        assert res["cells"].tolist() == r["cells"].tolist()
        H.assert_attention_close(res["out"], r["out"])


def test_capacity_overflow_is_reported_not_written():
    wl = synth.workload("tiny")
    qsa = _qsa(wl, max_ctx=8)
    g = H.GpuLayer(qsa)
    pre = synth.prefill_tokens(wl, 0, 8)
    g.append(pre["k"][:6], pre["v"][:6], pre["idx"][:6])
    g.append(pre["k"][:3], pre["v"][:3], pre["idx"][:3])  # 9 > 8: rejected on the device
    assert g.state(clear=True) == (6, 0, 2)
    g.append(pre["k"][6:8], pre["v"][6:8], pre["idx"][6:8])
    assert g.state()[:2] == (8, 0)
    np.testing.assert_array_equal(g.buf["k_cache"].cpu().numpy(), pre["k"])


def test_gather_materialises_compact_kv():
    wl = synth.workload("tiny")
    qsa, g, ref = _prefilled(wl)
    st = synth.step_inputs(wl, 0, 0)
    g.append(st["k"], st["v"], st["idx"])
    g.update()
    g.index_topk(st["q_idx"], st["w"])
    kc = torch.zeros(wl.max_cells, wl.n_kv_heads, wl.head_dim, dtype=torch.float16, device="cuda")
    vc = torch.zeros_like(kc)
    g.gather(kc, vc)
    res = g.fetch()
    nc = len(res["cells"])
    kk = g.buf["k_cache"].cpu().numpy()
    vv = g.buf["v_cache"].cpu().numpy()
    np.testing.assert_array_equal(kc[:nc].cpu().numpy(), kk[res["cells"]])
    np.testing.assert_array_equal(vc[:nc].cpu().numpy(), vv[res["cells"]])


def test_repeat_runs_are_bit_identical():
    wl = synth.workload("tiny")
    outs = []
    for _ in range(2):
        qsa, g, ref = _prefilled(wl)
        outs.append(g.step(synth.step_inputs(wl, 0, 3)))
    for key in ("sel", "cells", "out", "scores"):
        np.testing.assert_array_equal(outs[0][key], outs[1][key])


def test_cuda_graph_replay_matches_eager():
    wl = synth.workload("tiny")
    qsa_a, ga, _ = _prefilled(wl)
    qsa_b, gb, _ = _prefilled(wl)
    steps = [synth.step_inputs(wl, 0, s) for s in range(wl.n_steps)]
    eager = [ga.step(st) for st in steps]
    # graph: inputs staged in fixed device buffers, one captured step replayed per token
    stage = {k: H.to_dev(v) for k, v in steps[0].items()}
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    o = gb.outs
    with torch.cuda.stream(s):
        with torch.cuda.graph(graph, stream=s):
            qsa_b.append_token(0, stage["k"], stage["v"], stage["idx"], stream=s)
            qsa_b.update_pooled_cache(0, stream=s)
            qsa_b.index_topk(0, stage["q_idx"], stage["w"], o["sel"], o["n_sel"], gb.scores, stream=s)
            qsa_b.gather_kv(0, o["sel"], o["n_sel"], o["cells"], o["n_cells"], stream=s)
            qsa_b.sparse_attend(0, stage["q"], o["cells"], o["n_cells"], o["out"], stream=s)
    torch.cuda.synchronize()
    # capture does not execute: the state is still the prefill
    assert gb.state()[0] == wl.n_prefill
    for st, want in zip(steps, eager):
        for k, v in st.items():
            stage[k].copy_(H.to_dev(v))
        graph.replay()
        got = gb.fetch()
        for key in ("sel", "cells", "out"):
            np.testing.assert_array_equal(got[key], want[key])


# ----------------------------------------------------------------------------- full size

@pytest.mark.slow
@pytest.mark.parametrize("wl_name", ["ctx64k", "ctx128k", "ctx256k_12l"])
def test_full_size_layer_step(wl_name):
    """One layer at the pages' context length, launched like the bench: pooled cache
    (sampled rows), selection on the oracle's own pooled table, attention on the oracle's
    cells, and the end-to-end chain."""
    wl = synth.workload(wl_name)
    n0 = wl.n_prefill
    qsa = _qsa(wl)
    g = H.GpuLayer(qsa)
    shape = O.QsaShape.of(wl)
    pre = synth.prefill_tokens(wl, 0)
    g.append(pre["k"], pre["v"], pre["idx"])
    g.update()
    st = synth.step_inputs(wl, 0, 0)
    res = g.step(st)
    n = n0 + 1
    raw_idx = np.concatenate([pre["idx"], st["idx"][None]])
    ref_pooled = O.pooled_cache_full(raw_idx, n, shape)
    rng = np.random.default_rng(0)
    rows = np.unique(np.concatenate([rng.choice(n // 4, 2000, replace=False), np.arange(n // 4 - 8, n // 4)]))
    gp = g.pooled_rows(0, n // 4)
    H.assert_pooled_close(gp[rows], ref_pooled[rows])
    ref_scores = O.block_scores(ref_pooled, st["q_idx"], st["w"], n, shape)
    flips = H.selection_mismatch(res["sel"], ref_scores, shape.k_blocks, H.CHAIN_GAP_REL)
    # stage-isolated selection: the oracle's f16 table in the GPU cache
    g.buf["pooled_cache"][: n // 4] = H.to_dev(ref_pooled)
    g.index_topk(st["q_idx"], st["w"])
    iso = g.fetch()
    assert H.selection_mismatch(iso["sel"], ref_scores, shape.k_blocks, H.TIE_GAP_REL) <= 2
    # attention over the oracle's cells
    ref_sel = O.topk_blocks(ref_scores, shape.k_blocks)
    ref_cells = O.expand_cells(ref_sel, n)
    k_all = np.concatenate([pre["k"], st["k"][None]])
    v_all = np.concatenate([pre["v"], st["v"][None]])
    ref_out = O.sparse_attention(st["q"], k_all, v_all, ref_cells, shape)
    cells_d = torch.zeros(wl.max_cells, dtype=torch.int32, device="cuda")
    cells_d[: len(ref_cells)] = H.to_dev(ref_cells.astype(np.int32))
    g.attend(st["q"], cells_d, torch.tensor([len(ref_cells)], dtype=torch.int32, device="cuda"))
    H.assert_attention_close(g.fetch()["out"], ref_out)
    # the chain's own output, always: over the oracle's cells when the selections agree,
    # else the oracle attends over the GPU's cells
    gpu_cells = O.expand_cells(res["sel"], n)
    chain_ref = ref_out if np.array_equal(gpu_cells, ref_cells) else O.sparse_attention(
        st["q"], k_all, v_all, gpu_cells, shape)
    H.assert_attention_close(res["out"], chain_ref)
    H.record_chain(wl_name, 0, flips)
    print(f"{wl_name}: n={n} cells={len(ref_cells)} chain flips={flips}")
    assert g.state() == (n, n // 4, 0)


def test_attend_selected_equals_oracle_chain_every_step():
    """Cell expansion fused into attention: same result as the oracle's cells -> attention."""
    wl = synth.workload("tiny")
    qsa, g, ref = _prefilled(wl)
    for step in range(wl.n_steps):
        st = synth.step_inputs(wl, 0, step)
        g.append(st["k"], st["v"], st["idx"])
        g.update()
        g.index_topk(st["q_idx"], st["w"])
        g.attend_selected(st["q"])
        res = g.fetch()
        r = ref.decode_step(st["k"], st["v"], st["idx"], st["q_idx"], st["w"], st["q"])
        gpu_cells = O.expand_cells(res["sel"], ref.n)
        H.assert_attention_close(res["out"], _ref_attention_over(gpu_cells, r, st, ref, wl))
    assert g.state()[2] == 0


@pytest.mark.slow
def test_attend_selected_full_size_256k():
    """Fused expansion + attention on the oracle's selection at the 256k layer shape."""
    wl = synth.workload("ctx256k_12l")
    n = 255182
    qsa = _qsa(wl, max_ctx=n + 2)
    g = H.GpuLayer(qsa)
    pre = synth.prefill_tokens(wl, 0, n)
    g.append(pre["k"], pre["v"], pre["idx"])
    qsa.restore_layer(0, n, 0)
    shape = O.QsaShape.of(wl)
    st = synth.step_inputs(wl, 0, 0)
    sel = O.topk_blocks(synth.random_pooled(wl, 0, n // 4, salt=5)[:, 0].astype(np.float64), shape.k_blocks)
    g.outs["sel"][: len(sel)] = H.to_dev(sel.astype(np.int32))
    g.outs["n_sel"][0] = len(sel)
    g.attend_selected(st["q"])
    out = g.fetch()["out"]
    ref = O.sparse_attention(st["q"], pre["k"], pre["v"], O.expand_cells(sel, n), shape)
    H.assert_attention_close(out, ref)
    assert g.state()[2] == 0


def test_decode_append_equals_append_then_update():
    """The fused decode append gives the same caches and state as the two separate calls."""
    wl = synth.workload("tiny")
    qa, ga, _ = _prefilled(wl, n=1021, max_ctx=1100)
    qb, gb, _ = _prefilled(wl, n=1021, max_ctx=1100)
    for step in range(11):
        st = synth.step_inputs(wl, 0, step)
        ga.append(st["k"], st["v"], st["idx"])
        ga.update()
        gb.qsa.decode_append(0, H.to_dev(st["k"]), H.to_dev(st["v"]), H.to_dev(st["idx"]))
        assert ga.state() == gb.state()
    n = ga.state()[0]
    np.testing.assert_array_equal(ga.pooled_rows(0, n // 4), gb.pooled_rows(0, n // 4))
    for key in ("k_cache", "v_cache", "idx_cache"):
        np.testing.assert_array_equal(ga.buf[key].cpu().numpy(), gb.buf[key].cpu().numpy())
    # a lagging cache (several blocks behind) is caught up by the fused call as well
    pre = synth.prefill_tokens(wl, 0, 9, first=n)
    ga.append(pre["k"], pre["v"], pre["idx"])
    gb.append(pre["k"], pre["v"], pre["idx"])
    st = synth.step_inputs(wl, 0, 20)
    ga.append(st["k"], st["v"], st["idx"])
    ga.update()
    gb.qsa.decode_append(0, H.to_dev(st["k"]), H.to_dev(st["v"]), H.to_dev(st["idx"]))
    assert ga.state() == gb.state() and ga.state()[1] == ga.state()[0] // 4
    n = ga.state()[0]
    np.testing.assert_array_equal(ga.pooled_rows(0, n // 4), gb.pooled_rows(0, n // 4))


@pytest.mark.slow
def test_streaming_512_steps_12_layers():
    """The streaming workload: from the 256k prefill, 512 decode steps (qsa_decode_step, the
    append and pooled update fused into the scan launch) on each of the 12 layers (128
    block completions per layer). Every 128 steps the live pooled cache equals a
    full rebuild bit for bit; at steps 0, 127, 255, 383 and 511 the step's selection and
    attention match the oracle, whose pooled cache evolves incrementally every step."""
    wl = synth.workload("stream256k_12l")
    shape = O.QsaShape.of(wl)
    checks = {0, 127, 255, 383, 511}
    for layer in range(wl.n_layers):
        qsa = _qsa(wl)
        g = H.GpuLayer(qsa)
        ref = O.OracleLayer(shape, max_ctx=g.cfg.max_ctx)
        pre = synth.prefill_tokens(wl, layer)
        g.append(pre["k"], pre["v"], pre["idx"])
        g.update()
        ref.append_tokens(pre["k"], pre["v"], pre["idx"])
        ref.update_pooled_cache()
        del pre
        for step, st in enumerate(synth.step_inputs_range(wl, layer, 0, wl.n_steps)):
            d = {k: H.to_dev(x) for k, x in st.items()}   # the bench's call: qsa_decode_step
            qsa.decode_step(0, d["k"], d["v"], d["idx"], d["q_idx"], d["w"], d["q"], g.outs["sel"], g.outs["n_sel"],
                            g.outs["out"])
            ref.append_tokens(st["k"][None], st["v"][None], st["idx"][None])
            ref.update_pooled_cache()
            n = ref.n
            if step in checks:
                got = g.fetch()
                ref_scores = O.block_scores(ref.pooled.rows, st["q_idx"], st["w"], n, shape)
                H.selection_mismatch(got["sel"], ref_scores, shape.k_blocks, H.CHAIN_GAP_REL)
                cells = O.expand_cells(got["sel"], n)
                H.assert_attention_close(got["out"], O.sparse_attention(st["q"], ref.k, ref.v, cells, shape))
                rows = np.arange(max(0, n // 4 - 64), n // 4)
                H.assert_pooled_close(g.pooled_rows(0, n // 4)[rows], ref.pooled.rows[rows])
            if (step + 1) % 128 == 0:
                live = g.pooled_rows(0, n // 4)
                qsa.invalidate_pooled_cache(0, 0)
                g.buf["pooled_cache"].zero_()
                g.update()
                np.testing.assert_array_equal(g.pooled_rows(0, n // 4), live)
        assert g.state() == (wl.n_prefill + wl.n_steps, (wl.n_prefill + wl.n_steps) // 4, 0)
        del g, qsa, ref
        torch.cuda.empty_cache()


def test_decode_step_call_equals_separate_calls():
    """qsa_decode_step (the four launches in one ABI call) gives bit-identical results to
    qsa_decode_append + qsa_index_topk + qsa_sparse_attend_selected; qsa_n_ctx and
    qsa_get_device_status report the device state."""
    wl = synth.workload("tiny")
    layers = []
    for _ in range(2):
        qsa = _qsa(wl)
        g = H.GpuLayer(qsa)
        pre = synth.prefill_tokens(wl, 0, 1021)
        g.append(pre["k"], pre["v"], pre["idx"])
        g.update()
        layers.append((qsa, g))
    (qa, ga), (qb, gb) = layers
    for step in range(6):
        st = synth.step_inputs(wl, 0, step)
        d = {k: H.to_dev(x) for k, x in st.items()}
        qa.decode_step(0, d["k"], d["v"], d["idx"], d["q_idx"], d["w"], d["q"], ga.outs["sel"], ga.outs["n_sel"],
                       ga.outs["out"])
        qb.decode_append(0, d["k"], d["v"], d["idx"])
        gb.index_topk(st["q_idx"], st["w"])
        gb.attend_selected(st["q"])
        torch.cuda.synchronize()
        na, nb = int(ga.outs["n_sel"][0]), int(gb.outs["n_sel"][0])
        assert na == nb
        assert torch.equal(ga.outs["sel"][:na], gb.outs["sel"][:nb])
        assert torch.equal(ga.outs["out"], gb.outs["out"])
        assert qa.n_ctx(0) == 1021 + step + 1
    assert qa.device_status() == 0
    # a stale pooled cache is reported through the device status
    qa.invalidate_pooled_cache(0, 10)
    qa.index_topk(0, H.to_dev(st["q_idx"]), H.to_dev(st["w"]), ga.outs["sel"], ga.outs["n_sel"])
    assert qa.device_status() == 3  # QSA_ERR_STATE
