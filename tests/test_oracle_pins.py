"""Pins of the CPU oracle against facts fixed outside it.

Each test checks the oracle against something other than itself: values the
pages print (tests/golden/pages_constants.json), closed forms, independent
formulations (complex exponentials, rank counting, exact fractions), a library
routine (torch's scaled_dot_product_attention in float64) and invariants the
pages state (the incremental cache equals a full recompute; a selection that
covers every block equals dense attention). A plausible mistake in the oracle
(a dropped term, a wrong sign, position or index) fails at least one of them.
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import synth
from oracle import qsa_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
SMALL = O.QsaShape(d_idx=16, n_idx_heads=3, top_k_tokens=16, n_q_heads=4, n_kv_heads=2, head_dim=8)


def _pages():
    with open(os.path.join(GOLDEN, "pages_constants.json")) as f:
        return json.load(f)


# ---------------------------------------------------------------- f16 storage

def test_f16_rounding_is_direct_nearest_even():
    x = np.array([1 + 2**-11, 1 + 3 * 2**-11, 1 + 2**-11 + 2**-40, -(1 + 2**-11)])
    got = O.to_f16(x).astype(np.float64)
    # ties go to the even mantissa; a value just above a tie rounds up (no double rounding)
    assert got.tolist() == [1.0, 1 + 2**-9, 1 + 2**-10, -1.0]


# ---------------------------------------------------------------- RoPE

def test_rope_equals_complex_exponential():
    rng = np.random.default_rng(1)
    d, base = 32, 10000.0
    x = rng.standard_normal((5, d))
    pos = np.array([0, 1, 7, 4096, 255181])
    z = x[:, : d // 2] + 1j * x[:, d // 2:]
    freq = np.power(base, -np.arange(0, d, 2, dtype=np.float64) / d)
    zr = z * np.exp(1j * pos[:, None] * freq[None, :])
    want = np.concatenate([zr.real, zr.imag], axis=1)
    np.testing.assert_allclose(O.rope(x, pos, base), want, rtol=0, atol=1e-12)


def test_rope_equals_rotate_half_form():
    rng = np.random.default_rng(2)
    d = 16
    x = rng.standard_normal(d)
    inv = 1.0 / (10000.0 ** (np.arange(0, d, 2) / d))
    emb = np.concatenate([inv, inv]) * 9
    rot = np.concatenate([-x[d // 2:], x[: d // 2]])
    want = x * np.cos(emb) + rot * np.sin(emb)
    np.testing.assert_allclose(O.rope(x, 9, 10000.0), want, atol=1e-13)


def test_rope_identity_norms_and_relative_position():
    rng = np.random.default_rng(3)
    a, b = rng.standard_normal(64), rng.standard_normal(64)
    np.testing.assert_array_equal(O.rope(a, 0, 1e4), a)
    ra = O.rope(a, 1234, 1e4)
    pair = lambda v: v[:32] ** 2 + v[32:] ** 2
    np.testing.assert_allclose(pair(ra), pair(a), rtol=1e-12)
    for m, n in [(5, 5), (100, 3), (4 * 63000, 255180)]:
        lhs = O.rope(a, m, 1e4) @ O.rope(b, n, 1e4)
        rhs = a @ O.rope(b, n - m, 1e4)
        assert abs(lhs - rhs) <= 1e-9 * (np.abs(a).sum() * np.abs(b).sum())


def test_rope_interleaved_equals_complex_exponential_per_adjacent_pair():
    """GPT-J pairs: z_i = x[2i] + j*x[2i+1] times exp(j*pos*base^(-2i/d)), written out pair by pair."""
    rng = np.random.default_rng(31)
    d, base, pos = 12, 500.0, 37
    x = rng.standard_normal(d)
    want = np.empty(d)
    for i in range(d // 2):
        z = complex(x[2 * i], x[2 * i + 1]) * np.exp(1j * pos * base ** (-2.0 * i / d))
        want[2 * i], want[2 * i + 1] = z.real, z.imag
    np.testing.assert_allclose(O.rope(x, pos, base, interleaved=True), want, rtol=0, atol=1e-13)


def test_rope_partial_rotates_leading_dims_only():
    """rope_dims R < d: the first R dims turn like a full R-wide RoPE, the rest are copied."""
    rng = np.random.default_rng(32)
    x = rng.standard_normal((3, 64))
    pos = np.array([1, 999, 262143])
    for inter in (False, True):
        got = O.rope(x, pos, 1e4, rope_dims=16, interleaved=inter)
        np.testing.assert_array_equal(got[:, 16:], x[:, 16:])
        np.testing.assert_array_equal(got[:, :16], O.rope(x[:, :16], pos, 1e4, interleaved=inter))
    # written out: pair (i, i+8) of the 16 rotary dims turns by pos * base^(-2i/16)
    i = 5
    z = complex(x[1, i], x[1, i + 8]) * np.exp(1j * 999 * 1e4 ** (-2.0 * i / 16))
    got = O.rope(x[1], 999, 1e4, rope_dims=16)
    assert abs(got[i] - z.real) < 1e-12 and abs(got[i + 8] - z.imag) < 1e-12
    with pytest.raises(ValueError):
        O.rope(x, 1, 1e4, rope_dims=15)


def test_rope_switches_keep_identity_norms_and_relative_position():
    rng = np.random.default_rng(33)
    a, b = rng.standard_normal(64), rng.standard_normal(64)
    for dims, inter in [(0, True), (32, False), (32, True), (2, False)]:
        f = lambda v, p: O.rope(v, p, 1e4, rope_dims=dims, interleaved=inter)
        np.testing.assert_array_equal(f(a, 0), a)
        assert abs(np.linalg.norm(f(a, 4321)) - np.linalg.norm(a)) < 1e-12
        for m, n in [(7, 7), (100, 3), (4 * 63000, 255180)]:
            assert abs(f(a, m) @ f(b, n) - a @ f(b, n - m)) <= 1e-9 * (np.abs(a).sum() * np.abs(b).sum())


def test_query_position_table():
    """Query position floor(stride*(n-1)/4), by hand: token n-1, or the index of its block."""
    assert [O.query_position(n) for n in range(1, 10)] == [0, 1, 2, 3, 4, 5, 6, 7, 8]
    assert [O.query_position(n, 1) for n in range(1, 10)] == [0, 0, 0, 0, 1, 1, 1, 1, 2]
    assert [O.query_position(n, 2) for n in range(1, 10)] == [0, 0, 1, 1, 2, 2, 3, 3, 4]
    assert O.block_position(np.array([0, 1, 5])).tolist() == [0, 4, 20]
    assert O.block_position(np.array([0, 1, 5]), 1, 3).tolist() == [3, 4, 8]


def test_block_position_switches_on_periodic_keys():
    """With every block holding the same 4 raw keys, summaries differ only by position:
    offset 4 at block b is the default summary of block b+1; stride 8 at b is the default of 2b."""
    rng = np.random.default_rng(34)
    d = 32
    one = rng.standard_normal((4, d)).astype(np.float16)
    raw = np.tile(one, (40, 1))
    base = O.QsaShape(d, 1, 8, 1, 1, 8)
    dflt = O.pooled_cache_full(raw, 160, base)
    off4 = O.pooled_cache_full(raw, 160, O.QsaShape(d, 1, 8, 1, 1, 8, rope_pos_offset=4))
    st8 = O.pooled_cache_full(raw, 80, O.QsaShape(d, 1, 8, 1, 1, 8, rope_pos_stride=8))
    np.testing.assert_array_equal(off4[:39], dflt[1:40])
    np.testing.assert_array_equal(st8[:20], dflt[0:40:2])
    # block domain (stride 1): the query's own block is at relative distance 0, so its dot
    # is the un-rotated q . r (up to the f16 rounding of the stored row)
    shape = O.QsaShape(d, 1, 8, 1, 1, 8, rope_pos_stride=1)
    raw2 = rng.standard_normal((4 * 30, d)).astype(np.float16)
    q = rng.standard_normal((1, d)).astype(np.float16)
    n = 4 * 30                                    # query token 119 sits in block 29
    pooled = O.pooled_cache_full(raw2, n, shape)
    r = O.rms_normalize(O.mean_pool(raw2[116:120]), shape.rms_eps)
    qr = float(q[0].astype(np.float64) @ r)
    dot29 = float(pooled[29].astype(np.float64) @ O.indexer_query(q, n, shape)[0])
    assert abs(dot29 - qr) <= 2e-3 * np.abs(q[0].astype(np.float64)).sum() * np.abs(r).max()


# ---------------------------------------------------------------- pool + RMS norm

def test_mean_pool_is_exact_mean():
    rng = np.random.default_rng(4)
    raw = rng.standard_normal((4, 8)).astype(np.float16)
    got = O.mean_pool(raw)
    for j in range(8):
        exact = sum(Fraction(float(raw[i, j])) for i in range(4)) / 4
        assert Fraction(float(got[j])) == exact
    u = rng.standard_normal(8).astype(np.float16)
    np.testing.assert_array_equal(O.mean_pool(np.stack([u] * 4)), u.astype(np.float64))


def test_rms_norm_closed_forms():
    rng = np.random.default_rng(5)
    m = rng.standard_normal(128) * 3
    eps = 1e-6
    r = O.rms_normalize(m, eps)
    ms = np.mean(m * m)
    assert abs(np.sum(r * r) - 128 * ms / (ms + eps)) < 1e-10
    np.testing.assert_allclose(O.rms_normalize(7.0 * m, 0.0), O.rms_normalize(m, 0.0), rtol=1e-13)
    c = np.full(8, 0.5)
    np.testing.assert_allclose(O.rms_normalize(c, eps), c / np.sqrt(0.25 + eps), rtol=1e-15)
    g = rng.random(128)
    np.testing.assert_allclose(O.rms_normalize(m, eps, g), r * g, rtol=1e-15)


# ---------------------------------------------------------------- incremental cache (COMMON-004)

def test_incremental_cache_equals_full_recompute():
    rng = np.random.default_rng(6)
    shape = O.QsaShape(64, 4, 64, 8, 1, 64)
    raw = rng.standard_normal((400, 64)).astype(np.float16)
    cache = O.PooledKeyCache(100, 64)
    n = 0
    for step in [1, 3, 4, 5, 17, 2, 1, 1, 1, 64, 100, 7]:
        n += step
        cache.update(raw, n, shape)
        full = O.pooled_cache_full(raw, n, shape)
        assert cache.n_pooled == n // 4
        np.testing.assert_array_equal(cache.rows[: n // 4], full)
    cache.invalidate(30)
    assert cache.n_pooled == 30
    cache.rows[30:] = 0
    cache.update(raw, n, shape)
    np.testing.assert_array_equal(cache.rows[: n // 4], O.pooled_cache_full(raw, n, shape))


def test_pooled_summary_of_constant_block():
    rng = np.random.default_rng(7)
    u = rng.standard_normal(16).astype(np.float16)
    raw = np.stack([u] * 8)             # blocks 0 and 1, every key equal to u
    p = O.pooled_summaries(raw, 0, 2, SMALL)
    uu = u.astype(np.float64)
    r = uu / np.sqrt(np.mean(uu * uu) + SMALL.rms_eps)
    for b in (0, 1):
        z = (r[:8] + 1j * r[8:]) * np.exp(1j * 4 * b * np.power(1e4, -np.arange(0, 16, 2) / 16))
        want = np.concatenate([z.real, z.imag])
        np.testing.assert_allclose(p[b].astype(np.float64), want, rtol=0, atol=2e-3)


# ---------------------------------------------------------------- indexer scores

def test_scores_match_relative_complex_form():
    """s_b from the complex form: <RoPE(q, n-1), RoPE(r, 4b)> = Re sum conj(zq) zr e^{j(4b-n+1)theta}."""
    rng = np.random.default_rng(8)
    shape = SMALL
    d, H = shape.d_idx, shape.n_idx_heads
    n = 4 * 9 + 2
    raw = rng.standard_normal((n, d)).astype(np.float16)
    pooled = O.pooled_cache_full(raw, n, shape)
    q = rng.standard_normal((H, d)).astype(np.float16)
    w = np.array([0.25, 0.0, 1.5])
    got = O.block_scores(pooled, q, w, n, shape)
    assert got.shape == (n // 4,)
    theta = np.power(1e4, -np.arange(0, d, 2) / d)
    for b in range(n // 4):
        # undo the block rotation on the stored f16 row to get r_b, then rotate by the offset
        p = pooled[b].astype(np.float64)
        zp = (p[: d // 2] + 1j * p[d // 2:]) * np.exp(-1j * 4 * b * theta)
        s = 0.0
        for h in range(H):
            zq = q[h, : d // 2].astype(np.float64) + 1j * q[h, d // 2:].astype(np.float64)
            dot = np.real(np.sum(np.conj(zq) * zp * np.exp(1j * (4 * b - (n - 1)) * theta)))
            s += w[h] * max(dot, 0.0)
        assert abs(got[b] - s / np.sqrt(d)) <= 1e-10 * (1 + abs(s))


def test_scores_properties():
    rng = np.random.default_rng(9)
    shape = SMALL
    n = 4 * 20 + 3
    pooled = rng.standard_normal((n // 4, 16)).astype(np.float16)
    q = rng.standard_normal((3, 16)).astype(np.float16)
    w = rng.random(3)
    s = O.block_scores(pooled, q, w, n, shape)
    assert np.all(s >= 0)
    # positive homogeneity in the weights and linearity over heads
    np.testing.assert_allclose(O.block_scores(pooled, q, 3 * w, n, shape), 3 * s, rtol=1e-13)
    parts = sum(O.block_scores(pooled, q, np.eye(3)[h] * w[h], n, shape) for h in range(3))
    np.testing.assert_allclose(parts, s, rtol=1e-12)
    # a head whose query is negated keeps only the dots the other sign dropped
    s_pos = O.block_scores(pooled, q, np.array([1.0, 0, 0]), n, shape)
    qn = q.copy()
    qn[0] = -qn[0]
    s_neg = O.block_scores(pooled, qn, np.array([1.0, 0, 0]), n, shape)
    dots_abs = np.abs(pooled.astype(np.float64) @ O.rope(q[0].astype(np.float64), n - 1, 1e4))
    np.testing.assert_allclose(s_pos + s_neg, dots_abs / 4.0, rtol=1e-12)


def test_needle_blocks_are_selected():
    """Blocks whose keys point along the rotated query must win the top-k (pos(b)=4b, query n-1)."""
    rng = np.random.default_rng(10)
    shape = O.QsaShape(d_idx=64, n_idx_heads=2, top_k_tokens=12, n_q_heads=2, n_kv_heads=1, head_dim=16)
    n = 4 * 200 + 1
    raw = rng.standard_normal((n, 64)).astype(np.float16)
    q = rng.standard_normal((2, 64)).astype(np.float16)
    needles = [3, 77, 150]
    for b in needles:
        # r_b = RoPE(q_0, (n-1) - 4b) so that RoPE(r_b, 4b) = RoPE(q_0, n-1)
        key = O.rope(q[0].astype(np.float64), (n - 1) - 4 * b, 1e4)
        raw[4 * b:4 * b + 4] = key.astype(np.float16)
    pooled = O.pooled_cache_full(raw, n, shape)
    s = O.block_scores(pooled, q, np.array([1.0, 0.0]), n, shape)
    sel = O.topk_blocks(s, 3)
    assert sel.tolist() == needles


# ---------------------------------------------------------------- top-k (COMMON-006 form)

def _rank_count_selection(s, k):
    """Brute force: b is selected iff fewer than k blocks beat it (higher score, or equal and lower index)."""
    B = len(s)
    out = []
    for b in range(B):
        beaten_by = sum(1 for c in range(B) if s[c] > s[b] or (s[c] == s[b] and c < b))
        if beaten_by < k:
            out.append(b)
    return out


@pytest.mark.parametrize("seed", range(6))
def test_topk_equals_rank_counting(seed):
    rng = np.random.default_rng(100 + seed)
    B = int(rng.integers(1, 90))
    s = np.round(rng.random(B) * 8) / 8        # coarse values force many exact ties
    k = int(rng.integers(1, 40))
    assert O.topk_blocks(s, k).tolist() == _rank_count_selection(s.tolist(), k)


def test_topk_ties_lower_index_and_small_b():
    s = np.array([1.0, 2.0, 2.0, 2.0, 0.5, 2.0])
    assert O.topk_blocks(s, 2).tolist() == [1, 2]
    assert O.topk_blocks(s, 5).tolist() == [0, 1, 2, 3, 5]
    assert O.topk_blocks(s, 6).tolist() == [0, 1, 2, 3, 4, 5]
    assert O.topk_blocks(s, 100).tolist() == list(range(6))
    assert O.topk_blocks(np.zeros(0), 4).tolist() == []
    with pytest.raises(ValueError):
        O.topk_blocks(np.array([1.0, np.nan]), 1)


# ---------------------------------------------------------------- cells

def test_cells_count_order_and_tail():
    for n, sel in [(0, []), (3, []), (4, [0]), (23, [0, 2, 4]), (26, [5])]:
        cells = O.expand_cells(np.array(sel, dtype=np.int64), n)
        assert len(cells) == 4 * len(sel) + n % 4
        assert np.all(np.diff(cells) > 0) and (len(cells) == 0 or cells[-1] < n)
        assert set(range(4 * (n // 4), n)) <= set(cells.tolist())


def test_pages_max_cells():
    pg = _pages()
    k_tokens = pg["indexer_top_k"]["value"]
    ratio = pg["compression_ratio"]["value"]
    assert ratio == O.BLOCK
    k = k_tokens // ratio
    # the worst case: at least k completed blocks and a tail of 3
    for n in pg["input_tokens"]["value"] + [255182, 255183, 255184]:
        n_cells = len(O.expand_cells(np.arange(min(k, n // 4)), n))
        assert n_cells <= pg["max_cells"]["value"]
    assert len(O.expand_cells(np.arange(k), 4 * 1000 + 3)) == pg["max_cells"]["value"]


def test_pages_kv_cache_size_matches_layer_shapes():
    """2 x Hkv x D x f16 per token and layer, over 12 QSA layers, gives the pages' 6,144 MiB at 262,144."""
    pg = _pages()
    wl = synth.workload("ctx256k_12l")
    per_tok = 2 * wl.n_kv_heads * wl.head_dim * 2 * pg["qsa_layers"]["value"]
    assert per_tok * pg["kv_cache_mib"]["ctx"] == pg["kv_cache_mib"]["normal_kv"] * 2**20


# ---------------------------------------------------------------- attention (COMMON-005)

def _dense_sdpa(q, k, v, shape):
    """torch scaled_dot_product_attention in float64 over all tokens (GQA by head grouping)."""
    qt = torch.from_numpy(np.asarray(q, np.float64)).reshape(1, shape.n_q_heads, 1, shape.head_dim)
    kt = torch.from_numpy(np.asarray(k, np.float64)).permute(1, 0, 2).unsqueeze(0)
    vt = torch.from_numpy(np.asarray(v, np.float64)).permute(1, 0, 2).unsqueeze(0)
    out = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, enable_gqa=True)
    return out.reshape(shape.n_q_heads, shape.head_dim).numpy()


def test_full_selection_equals_dense_attention():
    wl = synth.workload("tiny")
    shape = O.QsaShape.of(wl)
    layer = O.OracleLayer(shape, max_ctx=wl.max_ctx)
    n0 = 4 * shape.k_blocks - 2          # every block fits in the top-k
    pre = synth.prefill_tokens(wl, 0, n0)
    layer.append_tokens(pre["k"], pre["v"], pre["idx"])
    layer.update_pooled_cache()
    st = synth.step_inputs(wl, 0, 0)
    res = layer.decode_step(st["k"], st["v"], st["idx"], st["q_idx"], st["w"], st["q"])
    n = n0 + 1
    assert res["cells"].tolist() == list(range(n))
    want = _dense_sdpa(st["q"], layer.k[:n], layer.v[:n], shape)
    np.testing.assert_allclose(res["out"], want, rtol=0, atol=1e-12)


def test_attention_special_cases():
    rng = np.random.default_rng(11)
    shape = SMALL
    k = rng.standard_normal((20, 2, 8)).astype(np.float16)
    v = rng.standard_normal((20, 2, 8)).astype(np.float16)
    q = rng.standard_normal((4, 8)).astype(np.float16)
    out = O.sparse_attention(q, k, v, np.array([13]), shape)
    for i in range(4):
        np.testing.assert_array_equal(out[i], v[13, i // 2].astype(np.float64))
    k_same = np.broadcast_to(k[:1], k.shape)
    out = O.sparse_attention(q, k_same, v, np.array([1, 4, 9]), shape)
    for i in range(4):
        np.testing.assert_allclose(out[i], v[[1, 4, 9], i // 2].astype(np.float64).mean(0), atol=1e-14)


# ---------------------------------------------------------------- chain

def test_decode_chain_invariants_tiny():
    wl = synth.workload("tiny")
    shape = O.QsaShape.of(wl)
    layer = O.OracleLayer(shape, max_ctx=wl.max_ctx)
    pre = synth.prefill_tokens(wl, 0)
    layer.append_tokens(pre["k"], pre["v"], pre["idx"])
    layer.update_pooled_cache()
    for step in range(wl.n_steps):
        st = synth.step_inputs(wl, 0, step)
        res = layer.decode_step(st["k"], st["v"], st["idx"], st["q_idx"], st["w"], st["q"])
        n = wl.n_prefill + step + 1
        assert len(res["sel"]) == min(shape.k_blocks, n // 4)
        assert len(res["cells"]) == 4 * len(res["sel"]) + n % 4 <= wl.max_cells
        np.testing.assert_array_equal(layer.pooled.rows[: n // 4],
                                      O.pooled_cache_full(layer.idx, n, shape))
        assert np.all(np.isfinite(res["out"]))


def test_golden_tiny_chain_regression():
    """The oracle still reproduces the committed tiny-workload chain (tests/golden/make_golden.py)."""
    import importlib.util
    spec = importlib.util.spec_from_file_location("make_golden", os.path.join(GOLDEN, "make_golden.py"))
    mg = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mg)
    want = np.load(os.path.join(GOLDEN, "tiny_chain.npz"))
    got = mg.tiny_chain()
    assert sorted(want.files) == sorted(got)
    for key in want.files:
        np.testing.assert_allclose(got[key], want[key], rtol=1e-12, atol=0, err_msg=key)


# ---------------------------------------------------------------- multi-query step (speculative verify)

def _tokens(rng, shape, T):
    f16 = lambda *s: rng.standard_normal(s).astype(np.float16)
    return dict(k=f16(T, shape.n_kv_heads, shape.head_dim), v=f16(T, shape.n_kv_heads, shape.head_dim),
                idx=f16(T, shape.d_idx), q_idx=f16(T, shape.n_idx_heads, shape.d_idx),
                w=rng.random((T, shape.n_idx_heads)), q=f16(T, shape.n_q_heads, shape.head_dim))


@pytest.mark.parametrize("n0,T", [(97, 4), (98, 3), (100, 2), (101, 1), (4 * 9 + 2, 4)])
def test_multi_query_step_equals_sequential_decode(n0, T):
    """T queries verified in one step see exactly what T single-token steps would see."""
    rng = np.random.default_rng(n0 * 10 + T)
    shape = SMALL
    pre = _tokens(rng, shape, n0)
    a, b = O.OracleLayer(shape, 256), O.OracleLayer(shape, 256)
    for L in (a, b):
        L.append_tokens(pre["k"], pre["v"], pre["idx"])
        L.update_pooled_cache()
    x = _tokens(rng, shape, T)
    multi = a.multi_query_step(x["k"], x["v"], x["idx"], x["q_idx"], x["w"], x["q"])
    for t in range(T):
        one = b.decode_step(x["k"][t], x["v"][t], x["idx"][t], x["q_idx"][t], x["w"][t], x["q"][t])
        for key in ("sel", "cells", "scores", "out"):
            np.testing.assert_array_equal(multi[t][key], one[key])
        # causality: query t never sees a later token, and its own open tail is attended
        n_t = n0 + t + 1
        assert multi[t]["cells"].max() < n_t
        assert set(range(4 * (n_t // 4), n_t)) <= set(multi[t]["cells"].tolist())
    np.testing.assert_array_equal(a.pooled.rows, b.pooled.rows)


def test_rollback_recomputes_blocks_completed_by_rejected_tokens():
    """Tokens n0..n0+3 with n0 = 4m+2: token n0+1 completes block m. Rejecting it (keep n0+1
    tokens) must drop that summary, so later steps equal a layer that never saw it."""
    rng = np.random.default_rng(77)
    shape = SMALL
    n0 = 4 * 20 + 2
    pre = _tokens(rng, shape, n0)
    a, b = O.OracleLayer(shape, 256), O.OracleLayer(shape, 256)
    for L in (a, b):
        L.append_tokens(pre["k"], pre["v"], pre["idx"])
        L.update_pooled_cache()
    draft = _tokens(rng, shape, 4)
    a.multi_query_step(draft["k"], draft["v"], draft["idx"], draft["q_idx"], draft["w"], draft["q"])
    assert a.pooled.n_pooled == 21
    a.rollback(n0 + 1)                                # keep the first draft token only
    assert (a.n, a.pooled.n_pooled) == (n0 + 1, 20)
    b.decode_step(draft["k"][0], draft["v"][0], draft["idx"][0], draft["q_idx"][0], draft["w"][0], draft["q"][0])
    nxt = _tokens(rng, shape, 3)                      # different tokens at the rejected positions
    ra = a.multi_query_step(nxt["k"], nxt["v"], nxt["idx"], nxt["q_idx"], nxt["w"], nxt["q"])
    rb = b.multi_query_step(nxt["k"], nxt["v"], nxt["idx"], nxt["q_idx"], nxt["w"], nxt["q"])
    np.testing.assert_array_equal(a.pooled.rows[:a.n // 4], b.pooled.rows[:b.n // 4])
    for x, y in zip(ra, rb):
        np.testing.assert_array_equal(x["out"], y["out"])
        np.testing.assert_array_equal(x["sel"], y["sel"])
    # without the invalidation the stale summary of block 20 would differ from the fresh one
    stale = O.pooled_summaries(np.concatenate([pre["idx"], draft["idx"][:2]]), 20, 21, shape)
    assert not np.array_equal(stale[0], a.pooled.rows[20])


# ---------------------------------------------------------------- FP8 (e4m3) K/V cache

def test_e4m3_known_codes():
    """Values fixed by the e4m3 layout (bias 7, 3 mantissa bits, subnormals, S.1111.111 = NaN)."""
    known = {0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6, 0x38: 1.0, 0x39: 1.125,
             0x40: 2.0, 0x7E: 448.0, 0xB8: -1.0, 0xFE: -448.0}
    for c, v in known.items():
        assert O.e4m3_value(c) == v, hex(c)
    assert np.isnan(O.e4m3_value(0x7F)) and np.isnan(O.e4m3_value(0xFF))
    assert np.signbit(O.e4m3_value(0x80))
    finite = [c for c in range(256) if not np.isnan(O.e4m3_value(c))]
    assert len(finite) == 254
    np.testing.assert_array_equal(O.e4m3_encode(np.array([O.e4m3_value(c) for c in finite], np.float32)), finite)


def test_e4m3_encode_is_nearest_even_by_brute_force():
    rng = np.random.default_rng(41)
    x = np.concatenate([rng.standard_normal(3000) * s for s in (1e-3, 0.05, 1, 30, 300)]).astype(np.float32)
    vals = np.array([O.e4m3_value(c) for c in range(256)])
    codes = np.array([c for c in range(256) if not np.isnan(vals[c])])
    # midpoints between neighbours and values past the largest finite one
    grid = np.unique(np.abs(vals[codes]))
    x = np.concatenate([x, ((grid[:-1] + grid[1:]) / 2).astype(np.float32), np.float32([449, 500, -1e4])])
    got = O.e4m3_encode(x)
    for xi, gi in zip(x.astype(np.float64), got):
        if abs(xi) > 448:
            assert O.e4m3_value(gi) == np.sign(xi) * 448.0
            continue
        d = np.abs(vals[codes] - xi)
        best = codes[d == d.min()]
        best = best[(best & 0x80) == (0x80 if np.signbit(xi) else 0)] if len(best) > 1 else best
        if len(best) > 1:                       # a tie: the even mantissa wins
            best = best[(best & 1) == 0]
        assert O.e4m3_value(gi) == O.e4m3_value(best[0]), (xi, hex(gi), [hex(b) for b in best])


def test_kv_row_quantization_closed_forms():
    rng = np.random.default_rng(42)
    rows = rng.standard_normal((64, 4, 128)).astype(np.float16)
    rows[3, 1] = 0
    codes, scales = O.quantize_kv_rows(rows)
    assert codes.dtype == np.uint8 and scales.dtype == np.float32 and scales.shape == (64, 4)
    amax = np.abs(rows.astype(np.float32)).max(axis=-1)
    nz = amax > 0
    np.testing.assert_array_equal(scales[nz], (amax / np.float32(448))[nz])
    assert scales[3, 1] == 1.0 and not codes[3, 1].any()
    deq = O.dequantize_kv_rows(codes, scales)
    # the row maximum lands on +-448 exactly; every element within half a quantum
    np.testing.assert_array_equal(np.abs(deq).max(axis=-1)[nz], 448.0 * scales[nz].astype(np.float64))
    x = rows.astype(np.float64)
    bound = np.maximum(np.abs(x) * 2.0 ** -4, 2.0 ** -10 * scales[..., None])
    assert np.all(np.abs(deq - x) <= bound * (1 + 1e-6))


def test_fp8_layer_is_exact_on_e4m3_grid_rows():
    """Rows whose values lie on the e4m3 grid and whose largest magnitude is 448 quantise
    with scale 1 and no rounding, so the FP8 layer attends exactly like the f16 layer."""
    rng = np.random.default_rng(43)
    shape = SMALL
    grid = np.array([O.e4m3_value(c) for c in range(256) if not np.isnan(O.e4m3_value(c))])
    grid = grid[np.abs(grid) <= 8]
    n = 37
    k = rng.choice(grid, (n, shape.n_kv_heads, shape.head_dim)).astype(np.float16)
    v = rng.choice(grid, (n, shape.n_kv_heads, shape.head_dim)).astype(np.float16)
    k[:, :, 0] = 448.0
    v[:, :, 3] = -448.0
    idx = rng.standard_normal((n, shape.d_idx)).astype(np.float16)
    a, b = O.OracleLayer(shape, 64), O.OracleLayer(shape, 64, kv_fp8=True)
    for L in (a, b):
        L.append_tokens(k, v, idx)
    assert np.all(b.kv_scales[:n] == 1.0)
    q = rng.standard_normal((shape.n_q_heads, shape.head_dim)).astype(np.float16) * 0.01
    cells = np.arange(n)
    np.testing.assert_array_equal(a.attend(q, cells), b.attend(q, cells))


def _pooled_layers(rows, n, pooled_fp8):
    """An oracle layer whose pooled cache holds `rows` (f16) for a context of n tokens."""
    L = O.OracleLayer(SMALL, 4 * len(rows) + 8, pooled_fp8=pooled_fp8)
    L.n = n
    L.pooled.rows[: len(rows)] = rows
    L.pooled.n_pooled = n // 4
    return L


def test_pooled_fp8_is_exact_on_e4m3_grid_rows():
    """Summaries on the e4m3 grid whose largest magnitude is 448 quantise with scale 1 and
    no rounding: the 8-bit pooled keys then score exactly like the f16 ones (reading R13)."""
    rng = np.random.default_rng(51)
    grid = np.array([O.e4m3_value(c) for c in range(256) if not np.isnan(O.e4m3_value(c))])
    grid = grid[np.abs(grid) <= 8]
    rows = rng.choice(grid, (20, SMALL.d_idx)).astype(np.float16)
    rows[:, 2] = 448.0
    codes, scales = O.pooled_fp8_rows(rows)
    assert np.all(scales == 1.0)
    np.testing.assert_array_equal(O.dequantize_kv_rows(codes, scales), rows.astype(np.float64))
    q_idx = rng.standard_normal((SMALL.n_idx_heads, SMALL.d_idx)).astype(np.float16)
    w = rng.random(SMALL.n_idx_heads).astype(np.float32)
    a, b = _pooled_layers(rows, 81, False), _pooled_layers(rows, 81, True)
    np.testing.assert_array_equal(a.scores(q_idx, w), b.scores(q_idx, w))


def test_pooled_fp8_scores_within_the_quantisation_bound():
    """Every element moves by at most 2^-4 of itself (or half a subnormal quantum), so a
    score moves by at most sum_h w_h * sum_e |q~_he| * bound_e / sqrt(d); and the scores
    use code * scale, not the f16 rows (a plain reading of R13 against R12's rule)."""
    rng = np.random.default_rng(52)
    rows = rng.standard_normal((40, SMALL.d_idx)).astype(np.float16)
    q_idx = rng.standard_normal((SMALL.n_idx_heads, SMALL.d_idx)).astype(np.float16)
    w = rng.random(SMALL.n_idx_heads).astype(np.float32)
    n = 4 * 40 + 1
    f16, f8 = _pooled_layers(rows, n, False), _pooled_layers(rows, n, True)
    s16, s8 = f16.scores(q_idx, w), f8.scores(q_idx, w)
    codes, scales = O.pooled_fp8_rows(rows)
    x = rows.astype(np.float64)
    bound = np.maximum(np.abs(x) * 2.0 ** -4, 2.0 ** -10 * scales[:, None].astype(np.float64))
    q = np.abs(O.indexer_query(q_idx, n, SMALL))                        # [H, d]
    limit = (bound @ q.T) @ w.astype(np.float64) / np.sqrt(SMALL.d_idx)  # [B]
    assert np.all(np.abs(s8 - s16) <= limit * (1 + 1e-9) + 1e-12)
    assert np.abs(s8 - s16).max() > 0   # the rows are not on the grid: the 8-bit scores differ
    # a needle row aligned with every head's query still wins under the 8-bit keys
    needle = O.indexer_query(q_idx, n, SMALL).sum(axis=0)
    rows2 = rows.copy()
    rows2[17] = (needle / np.abs(needle).max() * 4).astype(np.float16)
    f8b = _pooled_layers(rows2, n, True)
    assert 17 in O.topk_blocks(f8b.scores(q_idx, w), 1)


# ---------------------------------------------------------------- seeded inputs

@pytest.mark.parametrize("first", [250, 258048 - 255181 - 5])   # the second range crosses a chunk boundary
def test_step_inputs_range_equals_single_steps(first):
    """The range draw returns exactly what one call per step returns (position-keyed chunks)."""
    wl = synth.workload("stream256k_12l")
    rng_steps = synth.step_inputs_range(wl, 3, first, 12)
    for i, got in enumerate(rng_steps):
        want = synth.step_inputs(wl, 3, first + i)
        assert got.keys() == want.keys()
        for k in want:
            np.testing.assert_array_equal(got[k], want[k])


# ---------------------------------------------------------------- context-parallel decomposition

def _cp_layer(seed, n, shape, extra=4):
    rng = np.random.default_rng(seed)
    L = O.OracleLayer(shape, max_ctx=n + extra)
    L.append_tokens(rng.standard_normal((n, shape.n_kv_heads, shape.head_dim)).astype(np.float16),
                    rng.standard_normal((n, shape.n_kv_heads, shape.head_dim)).astype(np.float16),
                    rng.standard_normal((n, shape.d_idx)).astype(np.float16))
    L.update_pooled_cache()
    q_idx = rng.standard_normal((shape.n_idx_heads, shape.d_idx)).astype(np.float16)
    w = rng.random(shape.n_idx_heads)
    q = rng.standard_normal((shape.n_q_heads, shape.head_dim)).astype(np.float16)
    return L, q_idx, w, q


def _cp_step(L, starts, q_idx, w, q):
    """The sharded step over layer L's caches, shards starting at the given block-aligned tokens."""
    n, shape = L.n, L.shape
    bounds = list(starts) + [n]
    cand_s, cand_b = [], []
    for r in range(len(starts)):
        b0, b1 = bounds[r] // 4, bounds[r + 1] // 4        # the last shard's open tail has no block
        s, b = O.shard_candidates(L.pooled.rows[b0:b1], b0, q_idx, w, n, shape)
        cand_s.append(s)
        cand_b.append(b)
    sel = O.merge_candidates(cand_s, cand_b, shape.k_blocks)
    parts = []
    for r in range(len(starts)):
        mine = sel[(sel >= bounds[r] // 4) & (sel < bounds[r + 1] // 4)]
        cells = O.expand_cells(mine, 4 * (bounds[r + 1] // 4))          # no tail ...
        if r == len(starts) - 1:                                            # ... except on the last shard
            cells = O.expand_cells(mine, n)
        parts.append(O.attention_partial(q, L.k, L.v, cells, shape))
    return sel, O.merge_partials(parts)


@pytest.mark.parametrize("starts", [[0], [0, 400], [0, 128, 132], [0, 4, 200, 204, 500], [0, 700]])
def test_context_parallel_step_equals_single_device(starts):
    shape = O.QsaShape(d_idx=32, n_idx_heads=3, top_k_tokens=64, n_q_heads=4, n_kv_heads=2, head_dim=16)
    n = 4 * 180 + 3
    L, q_idx, w, q = _cp_layer(len(starts) * 7 + starts[-1], n, shape)
    sel, out = _cp_step(L, starts, q_idx, w, q)
    ref_sel = O.topk_blocks(O.block_scores(L.pooled.rows, q_idx, w, n, shape), shape.k_blocks)
    np.testing.assert_array_equal(sel, ref_sel)
    ref_out = O.sparse_attention(q, L.k, L.v, O.expand_cells(ref_sel, n), shape)
    np.testing.assert_allclose(out, ref_out, rtol=0, atol=1e-12)


def test_candidate_merge_keeps_ties_to_the_lower_block():
    # equal scores across shards: the lower block wins, exactly as in one list
    got = O.merge_candidates([np.array([5.0, 3.0]), np.array([5.0, 3.0]), np.array([], float)],
                             [np.array([2, 7]), np.array([12, 20]), np.array([], np.int64)], 3)
    assert got.tolist() == [2, 7, 12]
    got = O.merge_candidates([np.array([1.0]), np.array([1.0, 1.0])], [np.array([9]), np.array([10, 11])], 2)
    assert got.tolist() == [9, 10]


def test_lse_merge_over_any_cell_partition():
    shape = O.QsaShape(d_idx=32, n_idx_heads=3, top_k_tokens=64, n_q_heads=4, n_kv_heads=2, head_dim=16)
    L, _, _, q = _cp_layer(99, 300, shape)
    cells = np.arange(300)
    rng = np.random.default_rng(3)
    owner = rng.integers(0, 4, size=300)                  # shard 3 may own nothing
    owner[owner == 3] = 2
    parts = [O.attention_partial(q, L.k, L.v, cells[owner == r], shape) for r in range(4)]
    assert np.all(np.isneginf(parts[3][1]))
    np.testing.assert_allclose(O.merge_partials(parts), O.sparse_attention(q, L.k, L.v, cells, shape),
                               rtol=0, atol=1e-12)


def test_context_parallel_over_decode_steps_with_a_growing_tail():
    """Tokens are appended to the last shard only; as its tail completes blocks they join the
    shard's candidates, and every step still equals the single-device step."""
    shape = O.QsaShape(d_idx=32, n_idx_heads=3, top_k_tokens=64, n_q_heads=4, n_kv_heads=2, head_dim=16)
    L, q_idx, w, q = _cp_layer(5, 4 * 150 + 1, shape, extra=16)
    rng = np.random.default_rng(8)
    starts = [0, 200, 400]
    for step in range(9):
        L.append_tokens(rng.standard_normal((1, shape.n_kv_heads, shape.head_dim)).astype(np.float16),
                        rng.standard_normal((1, shape.n_kv_heads, shape.head_dim)).astype(np.float16),
                        rng.standard_normal((1, shape.d_idx)).astype(np.float16))
        L.update_pooled_cache()
        q_idx = rng.standard_normal((shape.n_idx_heads, shape.d_idx)).astype(np.float16)
        sel, out = _cp_step(L, starts, q_idx, w, q)
        n = L.n
        ref_sel = O.topk_blocks(O.block_scores(L.pooled.rows, q_idx, w, n, shape), shape.k_blocks)
        np.testing.assert_array_equal(sel, ref_sel)
        ref_out = O.sparse_attention(q, L.k, L.v, O.expand_cells(ref_sel, n), shape)
        np.testing.assert_allclose(out, ref_out, rtol=0, atol=1e-12)
