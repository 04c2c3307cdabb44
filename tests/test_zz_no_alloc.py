"""qsa_sparse_attend_noalloc against qsa_sparse_attend.

The no-allocation entry point serves callers that cannot call cudaMalloc (for example
a plugin whose host runtime owns all device memory in its own arena, or a process
under a hard device-memory cap): they pass only their inputs and output, and the
split-KV scratch comes from a fixed array compiled into the library. This test calls
it through the C ABI twice in a row, with different queries and cell sets, and checks
each result against the regular entry point (which uses the layer workspace) on the
same inputs, within the attention tolerance the parity tests use. It runs last in the
collection order and also passes alone in a fresh process.
"""
import numpy as np
import pytest
import torch

import synth
from tests import gpu_harness as H

pytestmark = pytest.mark.gpu


def test_noalloc_attention_matches_workspace_entry_point_twice():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    H.ensure_library()
    import sparse_attention_decode_02_b200 as Q

    wl = synth.workload("ctx64k")
    n = 8192 + 3
    qsa = Q.Qsa(H.config_of(wl, max_ctx=n + 1))
    g = H.GpuLayer(qsa)
    pre = synth.prefill_tokens(wl, 0, n)
    g.append(pre["k"], pre["v"], pre["idx"])
    torch.cuda.synchronize()

    k_cache, v_cache = g.buf["k_cache"], g.buf["v_cache"]
    out_ref = torch.zeros(wl.n_q_heads, wl.head_dim, dtype=torch.float32, device="cuda")
    out_na = torch.zeros_like(out_ref)
    for call, n_cells in enumerate((wl.max_cells, 700)):
        cells = synth.random_cells(wl, 0, n, n_cells, salt=call)
        cells_d = torch.zeros(wl.max_cells, dtype=torch.int32, device="cuda")
        cells_d[:n_cells] = H.to_dev(cells)
        nc = torch.tensor([n_cells], dtype=torch.int32, device="cuda")
        q = H.to_dev(synth.step_inputs(wl, 0, 10 + call)["q"])
        qsa.sparse_attend(0, q, cells_d, nc, out_ref)
        out_na.fill_(float("nan"))
        Q.sparse_attend_noalloc(q, k_cache, v_cache, n, cells_d, nc, out_na, wl.n_q_heads, wl.n_kv_heads,
                                wl.head_dim, wl.top_k_tokens)
        torch.cuda.synchronize()
        ref = out_ref.cpu().numpy().astype(np.float64)
        got = out_na.cpu().numpy().astype(np.float64)
        assert np.all(np.isfinite(got)), f"call {call}: non-finite output"
        H.assert_attention_close(got, ref)

    # shapes beyond the fixed scratch are refused with a clear status, not launched
    with pytest.raises(Q.QsaError) as err:
        Q.sparse_attend_noalloc(q, k_cache, v_cache, n, cells_d, nc, out_na, 64, 8, 128, 4 * 8192)
    assert err.value.status == 2  # QSA_ERR_CAPACITY
