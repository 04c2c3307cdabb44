"""qsa_sparse_attend_noalloc against the oracle and against qsa_sparse_attend.

The no-allocation entry point serves callers that cannot call cudaMalloc (for example
a plugin whose host runtime owns all device memory in its own arena, or a process
under a hard device-memory cap): they pass only their inputs and output, and the
split-KV scratch comes from a fixed array compiled into the library. Each case calls it
through the C ABI several times in a row on one K/V cache, with different queries and
cell sets (all cells the shapes allow, one cell, none, a third of them), and checks every
result against the oracle attending over the same cells and against the regular entry
point (which uses the layer workspace) on the same inputs, within the attention
tolerance the parity tests use. The cases cover head_dim 64 and 128, query heads per KV
head 1, 2 and 8, and a shape whose partials end within 2% of the array's end. This file
runs last in the collection order and also passes alone in a fresh process.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import qsa_oracle as O
from tests import gpu_harness as H

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 1 << 20  # QSA_NOALLOC_SCRATCH_BYTES

# (workload, shape overrides, tokens in the cache)
CASES = [
    ("tiny", {}, 1027),                                                        # D 64, G 8
    ("tiny", dict(n_q_heads=8, n_kv_heads=8), 1027),                           # D 64, G 1
    ("ctx64k", dict(n_q_heads=16, n_kv_heads=8, top_k_tokens=512), 4099),      # D 128, G 2
    ("ctx64k", {}, 8195),                                                      # the 64k layer, G 8
    ("ctx64k", dict(n_q_heads=64, n_kv_heads=8, top_k_tokens=1980), 4099),     # near the array's end
]


def _scratch_bytes(wl, n_sms):
    """Bytes of the fixed array the entry point uses for these shapes: a 256-byte state
    block, the (max, sum) pair of every split and query head (256-byte aligned), and the
    partial outputs. The split size: the largest cell set spread over the SMs given to
    each KV head, rounded up to 8 cells, between 8 and 64."""
    max_cells = wl.max_cells
    per_head = max(1, n_sms // wl.n_kv_heads)
    cells = min(64, max(8, (-(-max_cells // per_head) + 7) // 8 * 8))
    n_splits = -(-max_cells // cells)
    ml = (n_splits * wl.n_q_heads * 8 + 255) // 256 * 256
    return 256 + ml + n_splits * wl.n_q_heads * wl.head_dim * 4


@pytest.mark.parametrize("wl_name,over,n", CASES)
def test_noalloc_attention_matches_oracle_and_workspace_entry_point(wl_name, over, n):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    H.ensure_library()
    import sparse_attention_decode_02_b200 as Q

    wl = synth.workload(wl_name, **over)
    shape = O.QsaShape.of(wl)
    n_sms = torch.cuda.get_device_properties(0).multi_processor_count
    need = _scratch_bytes(wl, n_sms)
    assert need <= SCRATCH_BYTES
    if wl.n_q_heads == 64:
        assert need > 0.98 * SCRATCH_BYTES, need

    qsa = Q.Qsa(H.config_of(wl, max_ctx=(n + 4) // 4 * 4))
    g = H.GpuLayer(qsa)
    pre = synth.prefill_tokens(wl, 0, n)
    g.append(pre["k"], pre["v"], pre["idx"])
    torch.cuda.synchronize()

    k_cache, v_cache = g.buf["k_cache"], g.buf["v_cache"]
    out_ref = torch.zeros(wl.n_q_heads, wl.head_dim, dtype=torch.float32, device="cuda")
    out_na = torch.zeros_like(out_ref)
    cells_d = torch.zeros(wl.max_cells, dtype=torch.int32, device="cuda")
    for call, n_cells in enumerate((wl.max_cells, 1, 0, wl.max_cells // 3)):
        cells = synth.random_cells(wl, 0, n, n_cells, salt=call)
        cells_d.zero_()
        cells_d[:n_cells] = H.to_dev(cells)
        nc = torch.tensor([n_cells], dtype=torch.int32, device="cuda")
        q_host = synth.step_inputs(wl, 0, 10 + call)["q"]
        q = H.to_dev(q_host)
        qsa.sparse_attend(0, q, cells_d, nc, out_ref)
        out_na.fill_(float("nan"))
        Q.sparse_attend_noalloc(q, k_cache, v_cache, n, cells_d, nc, out_na, wl.n_q_heads, wl.n_kv_heads,
                                wl.head_dim, wl.top_k_tokens)
        torch.cuda.synchronize()
        got = out_na.cpu().numpy().astype(np.float64)
        ref = out_ref.cpu().numpy().astype(np.float64)
        assert np.all(np.isfinite(got)), f"call {call}: non-finite output"
        if n_cells == 0:  # no cells: every output row is zero, as from the workspace entry point
            assert not got.any() and not ref.any(), f"call {call}: output of an empty cell set"
            continue
        H.assert_attention_close(got, O.sparse_attention(q_host, pre["k"], pre["v"], cells.astype(np.int64), shape))
        H.assert_attention_close(got, ref)

    # a negative cell count is read as no cells
    nc = torch.tensor([-5], dtype=torch.int32, device="cuda")
    out_na.fill_(float("nan"))
    Q.sparse_attend_noalloc(q, k_cache, v_cache, n, cells_d, nc, out_na, wl.n_q_heads, wl.n_kv_heads, wl.head_dim,
                            wl.top_k_tokens)
    torch.cuda.synchronize()
    assert not out_na.cpu().numpy().any()


def test_noalloc_refuses_shapes_beyond_the_array():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    H.ensure_library()
    import sparse_attention_decode_02_b200 as Q

    t = lambda *s, dt=torch.float16: torch.zeros(*s, dtype=dt, device="cuda")
    q, k, v = t(64, 128), t(16, 8, 128), t(16, 8, 128)
    cells, nc, out = t(32771, dt=torch.int32), t(1, dt=torch.int32), t(64, 128, dt=torch.float32)
    # 64 query heads over 8 KV heads with 8,192 selected blocks: partials beyond the array
    with pytest.raises(Q.QsaError) as err:
        Q.sparse_attend_noalloc(q, k, v, 16, cells, nc, out, 64, 8, 128, 4 * 8192)
    assert err.value.status == 2  # QSA_ERR_CAPACITY
    # the 1,980-token shape above fits; 2,048 tokens with the same heads does not
    assert _scratch_bytes(synth.workload("ctx64k", n_q_heads=64, n_kv_heads=8, top_k_tokens=2048),
                          torch.cuda.get_device_properties(0).multi_processor_count) > SCRATCH_BYTES
    with pytest.raises(Q.QsaError) as err:
        Q.sparse_attend_noalloc(q, k, v, 16, cells, nc, out, 64, 8, 128, 2048)
    assert err.value.status == 2
