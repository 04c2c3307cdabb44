"""The context-parallel exchange of one decode step over real collectives (gloo, CPU).

Each rank holds a contiguous, block-aligned shard of one layer's context (the last one
with the open tail) and computes, with the oracle, only what its shard allows: the
summaries of its own blocks, its local top-K candidates, and attention partials (o, lse)
over its selected cells. The candidates travel as fixed-size slots (K scores padded with
-inf, K block ids padded with -1) through all_gather; every rank merges them with the
selection rule; the partials travel through all_gather and merge exactly. Rank 0 checks
the result against the single-device definition. This pins the protocol the sharded
kernels follow (qsa_cp_index_candidates, qsa_cp_select, qsa_cp_attend_partial,
qsa_cp_merge; their GPU parity, with the shards emulated on one GPU, is in
test_gpu_context_parallel.py).
"""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

_WORKER = r"""
import json, os, sys
sys.path.insert(0, os.environ["QSA_ROOT"])
import numpy as np
import torch
import torch.distributed as dist
import synth
from oracle import qsa_oracle as O

dist.init_process_group("gloo")
rank, world = dist.get_rank(), dist.get_world_size()
wl = synth.workload("tiny")
shape = O.QsaShape.of(wl)
n = wl.n_prefill + 3
pre = synth.prefill_tokens(wl, 0, n)
st = synth.step_inputs(wl, 0, 0)
starts = [4 * ((r * (n // 4)) // world) for r in range(world)]
bounds = starts + [n]
t0, t1 = bounds[rank], bounds[rank + 1]
b0, b1 = t0 // 4, t1 // 4
K = shape.k_blocks

# this shard's summaries (its own raw keys only) and local candidates
mine_pooled = O.pooled_summaries(pre["idx"], b0, b1, shape)
s, b = O.shard_candidates(mine_pooled, b0, st["q_idx"], st["w"], n, shape)
slot_s = torch.full((K,), -float("inf"), dtype=torch.float64)
slot_b = torch.full((K,), -1, dtype=torch.int64)
slot_s[: len(s)] = torch.from_numpy(s)
slot_b[: len(b)] = torch.from_numpy(b)
all_s = [torch.empty_like(slot_s) for _ in range(world)]
all_b = [torch.empty_like(slot_b) for _ in range(world)]
dist.all_gather(all_s, slot_s)
dist.all_gather(all_b, slot_b)
keep = [y.numpy() >= 0 for y in all_b]
sel = O.merge_candidates([x.numpy()[k] for x, k in zip(all_s, keep)],
                         [y.numpy()[k] for y, k in zip(all_b, keep)], K)

# attention partials over this shard's selected cells (the tail only on the last shard)
mine = sel[(sel >= b0) & (sel < b1)]
cells = O.expand_cells(mine, n if rank == world - 1 else 4 * b1)
rows = np.zeros_like(pre["k"]), np.zeros_like(pre["v"])
rows[0][t0:t1], rows[1][t0:t1] = pre["k"][t0:t1], pre["v"][t0:t1]   # a shard sees only its rows
o, lse = O.attention_partial(st["q"], rows[0], rows[1], cells, shape)
all_o = [torch.empty(o.shape, dtype=torch.float64) for _ in range(world)]
all_l = [torch.empty(lse.shape, dtype=torch.float64) for _ in range(world)]
dist.all_gather(all_o, torch.from_numpy(o))
dist.all_gather(all_l, torch.from_numpy(lse))
out = O.merge_partials([(a.numpy(), l.numpy()) for a, l in zip(all_o, all_l)])

res = {"rank": rank, "n_cand": int(len(b)), "n_mine": int(len(mine))}
if rank == 0:
    full = O.pooled_cache_full(pre["idx"], n, shape)
    ref_sel = O.topk_blocks(O.block_scores(full, st["q_idx"], st["w"], n, shape), K)
    ref_out = O.sparse_attention(st["q"], pre["k"], pre["v"], O.expand_cells(ref_sel, n), shape)
    res.update(sel_equal=bool(np.array_equal(sel, ref_sel)), max_err=float(np.abs(out - ref_out).max()),
               n_sel=int(len(sel)))
with open(os.path.join(os.environ["QSA_OUT"], f"cp{rank}.json"), "w") as f:
    json.dump(res, f)
dist.destroy_process_group()
"""


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world", [2, 3])
def test_context_parallel_exchange(tmp_path, world):
    script = tmp_path / "cp_worker.py"
    script.write_text(_WORKER)
    env = dict(os.environ, QSA_ROOT=ROOT, QSA_OUT=str(tmp_path), CUDA_VISIBLE_DEVICES="", OMP_NUM_THREADS="1")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={world}",
           "--master-addr=127.0.0.1", f"--master-port={_free_port()}", str(script)]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-3000:]
    res = [json.loads((tmp_path / f"cp{i}.json").read_text()) for i in range(world)]
    head = res[0]
    assert head["sel_equal"] and head["n_sel"] == 64
    assert head["max_err"] <= 1e-12
    assert sum(x["n_mine"] for x in res) == 64            # every selected block attended exactly once
    assert all(0 < x["n_cand"] <= 64 for x in res)        # each shard sends at most K candidates
