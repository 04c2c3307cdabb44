"""Writes tiny_chain.npz: the oracle's decode chain on the tiny workload.

Calls only `oracle` and `synth`; run from the repository root:
    python tests/golden/make_golden.py
The stored values guard the oracle against unintended changes (any change to its
arithmetic must name, in its commit message, the passage that justifies it).
"""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import synth  # noqa: E402
from oracle import qsa_oracle as O  # noqa: E402


def tiny_chain():
    wl = synth.workload("tiny")
    shape = O.QsaShape.of(wl)
    layer = O.OracleLayer(shape, max_ctx=wl.max_ctx)
    pre = synth.prefill_tokens(wl, 0)
    layer.append_tokens(pre["k"], pre["v"], pre["idx"])
    layer.update_pooled_cache()
    out = {}
    for step in range(wl.n_steps):
        st = synth.step_inputs(wl, 0, step)
        res = layer.decode_step(st["k"], st["v"], st["idx"], st["q_idx"], st["w"], st["q"])
        out[f"sel{step}"] = res["sel"].astype(np.int32)
        out[f"out{step}"] = res["out"]
        out[f"top_scores{step}"] = np.sort(res["scores"])[-8:]
    out["pooled_last"] = layer.pooled.rows[: layer.n // 4]
    return out


if __name__ == "__main__":
    np.savez_compressed(os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_chain.npz"),
                        **tiny_chain())
    print("wrote tiny_chain.npz")
