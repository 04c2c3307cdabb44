"""GPU parity of the block selection alone (qsa_select_topk on caller-supplied scores)
against the oracle's top-k rule: the K largest, ties to the lower block index, ascending.

The score sets stress the radix select: spread-out scores, exact ties at the threshold
(thousands of equal keys, all-equal scores), high scores packed into neighbouring
blocks, negative scores, the extremes of the float range, signed zeros and NaN (ranked
lowest), and block counts around the CTA and group boundaries.
"""
import zlib

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


def _select(scores_f32, top_k_tokens, n_tail=0):
    import sparse_attention_decode_02_b200 as Q
    wl = synth.workload("ctx64k")
    n_blocks = len(scores_f32)
    n = 4 * n_blocks + n_tail
    qsa = Q.Qsa(H.config_of(wl, max_ctx=4 * n_blocks + 4, top_k_tokens=top_k_tokens))
    g = H.GpuLayer(qsa)
    qsa.restore_layer(0, n, n_blocks)
    sc = torch.zeros(qsa.cfg.max_ctx // 4, dtype=torch.float32, device="cuda")
    sc[:n_blocks] = torch.from_numpy(np.ascontiguousarray(scores_f32, dtype=np.float32)).cuda()
    o = g.outs
    qsa.select_topk(0, sc, o["sel"], o["n_sel"])
    torch.cuda.synchronize()
    ns = int(o["n_sel"][0])
    assert g.state()[2] == 0
    return o["sel"][:ns].cpu().numpy().astype(np.int64)


def _expected(scores_f32, k_blocks):
    s = np.asarray(scores_f32, np.float32).astype(np.float64)
    s = np.where(np.isnan(s), -1e300, s)   # NaN ranks below every f32 value
    s = np.where(s == 0.0, 0.0, s)         # -0 equals +0
    return O.topk_blocks(s, k_blocks)


def _rng(seed):
    return np.random.default_rng(seed)


CASES = {
    "normal_15447": lambda r: r.standard_normal(15447),
    "normal_63795": lambda r: r.standard_normal(63795),
    "uniform_positive_63795": lambda r: r.random(63795),
    "negative_only_40001": lambda r: -r.random(40001) - 1.0,
    # a few distinct values: thousands of exact ties at the threshold
    "quantised_63795": lambda r: np.round(r.random(63795), 1),
    "all_equal_50000": lambda r: np.full(50000, 0.25),
    # the top scores packed into neighbouring blocks: every flagged group is full
    "clustered_desc_63795": lambda r: np.concatenate([1000.0 - np.arange(20000) * 1e-2, r.random(43795)]),
    "clustered_equal_63795": lambda r: np.concatenate([np.ones(32768), r.random(31027) * 0.5]),
    "sparse_spikes_63795": lambda r: np.where(r.random(63795) < 0.004, 10 + r.random(63795), r.random(63795)),
}


@pytest.mark.parametrize("case", sorted(CASES))
@pytest.mark.parametrize("top_k_tokens", [2048, 4092, 64])
def test_select_matches_oracle_rule(case, top_k_tokens):
    s = CASES[case](_rng(zlib.crc32(case.encode()))).astype(np.float32)
    k = top_k_tokens // 4
    got = _select(s, top_k_tokens, n_tail=3)
    want = _expected(s, k)
    np.testing.assert_array_equal(got, want)


def test_select_signed_zero_and_nan():
    r = _rng(5)
    s = r.standard_normal(9000).astype(np.float32)
    s[r.random(9000) < 0.3] = 0.0
    s[r.random(9000) < 0.3] = -0.0
    s[r.random(9000) < 0.05] = np.nan
    s[s > 0] = 0.0                        # the K-th largest is a zero: ties among +0 and -0
    got = _select(s, 2048)
    np.testing.assert_array_equal(got, _expected(s, 512))
    s_nan = np.full(5000, np.nan, np.float32)
    s_nan[4000:] = -3.0                   # 1000 finite scores, then NaN fills the rest in order
    got = _select(s_nan, 4092)
    np.testing.assert_array_equal(got, _expected(s_nan, 1023))


def test_select_group_boundaries_and_ragged_tail():
    # block counts around multiples of the 32-block group, K just below the block count
    for n_blocks in (513, 543, 544, 545, 1055):
        s = _rng(n_blocks).random(n_blocks).astype(np.float32)
        np.testing.assert_array_equal(_select(s, 2048, n_tail=1), _expected(s, 512))


def test_select_extremes_of_float_range():
    r = _rng(11)
    s = (r.standard_normal(30000) * 1e30).astype(np.float32)
    s[::7] = np.float32(3.4e38)
    s[1::7] = np.float32(-3.4e38)
    s[2::11] = np.float32(1e-45)           # denormals
    s[3::13] = np.inf
    s[4::17] = -np.inf
    want = np.where(np.isinf(s), np.sign(s).astype(np.float64) * 1e300, s.astype(np.float64))
    got = _select(s, 4092)
    np.testing.assert_array_equal(got, O.topk_blocks(want, 1023))



# pairs of score sets of 63,795 blocks selected one after the other on the same layer:
# nothing of the first selection may leak into the second (same scale, another scale,
# another sign)
PAIRS = [("normal_63795", "normal_63795x1.01"), ("uniform_positive_63795", "uniform_positive_63795x1000"),
         ("uniform_positive_63795", "normal_63795"), ("clustered_desc_63795", "sparse_spikes_63795"),
         ("quantised_63795", "quantised_63795x0.5"), ("normal_63795", "negative_63795")]


def _scores_of(name):
    base, _, scale = name.partition("x")
    if base == "negative_63795":
        return (-_rng(3).random(63795) - 1.0).astype(np.float32)
    s = CASES[base](_rng(zlib.crc32(base.encode())))
    return (s * float(scale or 1.0)).astype(np.float32)


@pytest.mark.parametrize("first,second", PAIRS)
def test_select_after_a_previous_selection(first, second):
    import sparse_attention_decode_02_b200 as Q
    wl = synth.workload("ctx64k")
    n = 4 * 63795 + 2
    qsa = Q.Qsa(H.config_of(wl, max_ctx=n + 2))
    g = H.GpuLayer(qsa)
    qsa.restore_layer(0, n, n // 4)
    sc = torch.zeros(qsa.cfg.max_ctx // 4, dtype=torch.float32, device="cuda")
    o = g.outs
    for name in (first, second):
        s = _scores_of(name)
        sc[: len(s)] = torch.from_numpy(s).cuda()
        qsa.select_topk(0, sc, o["sel"], o["n_sel"])
        torch.cuda.synchronize()
        got = o["sel"][: int(o["n_sel"][0])].cpu().numpy().astype(np.int64)
        np.testing.assert_array_equal(got, _expected(s, wl.k_blocks), err_msg=name)
    assert g.state()[2] == 0
