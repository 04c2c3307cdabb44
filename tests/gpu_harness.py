"""Shared helpers of the GPU parity tests: set up a library layer from seeded inputs,
run the decode calls through the C ABI, and compare against the oracle with the
tolerances the tests use."""
from __future__ import annotations

import json
import os

import numpy as np
import torch

import synth
import sparse_attention_decode_02_b200 as Q
from sparse_attention_decode_02_b200 import build as qbuild

# Tolerances (see the design notes for their derivation)
POOLED_REL = 1e-3        # per element, relative to the row's largest |value|
SCORE_REL = 1e-5         # f32 scores vs float64 on identical f16 inputs, relative to max score
TIE_GAP_REL = 1e-6       # a selection may differ only where the oracle's score gap is below this
CHAIN_GAP_REL = 1e-4     # end-to-end chains (each side pooled its own f16 cache): f16-ulp flips
ATTN_REL = 2e-3          # attention output, relative to the head's largest |value|


def ensure_library():
    qbuild.build()
    return Q.load_library()


def config_of(wl: synth.Workload, max_ctx=None, n_layers=1, top_k_tokens=None, **rope) -> Q.QsaConfig:
    """Library config of a workload; `rope` takes the rope_* switches of make_config."""
    return Q.make_config(n_layers, max_ctx or wl.max_ctx, wl.d_idx, wl.n_idx_heads,
                         top_k_tokens or wl.top_k_tokens, wl.n_q_heads, wl.n_kv_heads, wl.head_dim,
                         wl.rope_base, wl.rms_eps, **rope)


def to_dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return t if dtype is None else t.to(dtype)


class GpuLayer:
    """One bound layer of a library context plus its per-step output buffers."""

    def __init__(self, qsa: Q.Qsa, layer: int = 0, gain=None):
        self.qsa, self.layer, self.cfg = qsa, layer, qsa.cfg
        self.buf = Q.alloc_layer(self.cfg)
        self.gain = None if gain is None else to_dev(np.asarray(gain, np.float32))
        qsa.bind_layer(layer, **self.buf, rms_gain=self.gain)
        self.outs = Q.alloc_step_outputs(self.cfg)
        self.scores = torch.zeros(self.cfg.max_ctx // 4, dtype=torch.float32, device="cuda")

    def append(self, k, v, idx):
        k, v, idx = to_dev(k), to_dev(v), to_dev(idx)
        if k.dim() == 2:
            self.qsa.append_token(self.layer, k, v, idx)
        else:
            self.qsa.append_tokens(self.layer, k, v, idx)

    def update(self):
        self.qsa.update_pooled_cache(self.layer)

    def index_topk(self, q_idx, w):
        o = self.outs
        self.qsa.index_topk(self.layer, to_dev(q_idx), to_dev(np.asarray(w, np.float32)), o["sel"], o["n_sel"],
                            self.scores)

    def gather(self, k_compact=None, v_compact=None):
        o = self.outs
        self.qsa.gather_kv(self.layer, o["sel"], o["n_sel"], o["cells"], o["n_cells"], k_compact, v_compact)

    def attend(self, q, cells=None, n_cells=None):
        o = self.outs
        self.qsa.sparse_attend(self.layer, to_dev(q), o["cells"] if cells is None else cells,
                               o["n_cells"] if n_cells is None else n_cells, o["out"])

    def attend_selected(self, q):
        o = self.outs
        self.qsa.sparse_attend_selected(self.layer, to_dev(q), o["sel"], o["n_sel"], o["out"])

    def step(self, st):
        """append -> pooled update -> scan + top-k -> cells -> attention (all on the stream)."""
        self.append(st["k"], st["v"], st["idx"])
        self.update()
        self.index_topk(st["q_idx"], st["w"])
        self.gather()
        self.attend(st["q"])
        return self.fetch()

    def fetch(self):
        torch.cuda.synchronize()
        o = self.outs
        ns, nc = int(o["n_sel"][0]), int(o["n_cells"][0])
        return {"sel": o["sel"][:ns].cpu().numpy().astype(np.int64),
                "cells": o["cells"][:nc].cpu().numpy().astype(np.int64),
                "out": o["out"].cpu().numpy().astype(np.float64),
                "scores": self.scores.cpu().numpy().astype(np.float64)}

    def state(self, clear=False):
        return self.qsa.read_layer_state(self.layer, clear=clear)

    def pooled_rows(self, b0, b1):
        torch.cuda.synchronize()
        return self.buf["pooled_cache"][b0:b1].cpu().numpy()


# ----------------------------------------------------------------------------- comparisons

def assert_pooled_close(gpu_rows, ref_rows):
    g = gpu_rows.astype(np.float64)
    r = ref_rows.astype(np.float64)
    scale = np.maximum(np.abs(r).max(axis=1, keepdims=True), 1e-6)
    err = np.abs(g - r) / scale
    assert err.max() <= POOLED_REL, f"pooled rows differ: max rel err {err.max():.3e}"


def selection_mismatch(gpu_sel, ref_scores, k_blocks, gap_rel):
    """Returns the number of blocks where the selections differ; asserts each one is a near-tie."""
    from oracle import qsa_oracle as O
    gpu_sel = np.asarray(gpu_sel, np.int64)
    ref_sel = O.topk_blocks(ref_scores, k_blocks)
    assert len(gpu_sel) == len(ref_sel), (len(gpu_sel), len(ref_sel))
    assert np.all(np.diff(gpu_sel) > 0), "selection must be strictly ascending"
    diff = set(gpu_sel.tolist()) ^ set(ref_sel.tolist())
    if diff:
        s_k = np.sort(ref_scores)[::-1][len(ref_sel) - 1]
        for b in diff:
            gap = abs(ref_scores[b] - s_k)
            assert gap <= gap_rel * abs(s_k), f"block {b}: score gap {gap:.3e} vs s_K {s_k:.6f}"
    return len(diff)


def assert_attention_close(gpu_out, ref_out):
    for i in range(ref_out.shape[0]):
        scale = max(np.abs(ref_out[i]).max(), 1e-6)
        err = np.abs(gpu_out[i] - ref_out[i]).max() / scale
        assert err <= ATTN_REL, f"head {i}: attention rel err {err:.3e}"


def record_chain(case: str, step: int, flips: int, **extra):
    """Appends one line (case, step, near-tie selection flips) to chain_flips.jsonl under
    $QSA_ARTIFACT_DIR when that variable is set: the per-context flip counts of the
    end-to-end chains, kept as a test artifact."""
    d = os.environ.get("QSA_ARTIFACT_DIR")
    if not d:
        return
    os.makedirs(d, exist_ok=True)
    with open(os.path.join(d, "chain_flips.jsonl"), "a") as f:
        f.write(json.dumps(dict(case=case, step=step, flips=flips, **extra)) + "\n")
