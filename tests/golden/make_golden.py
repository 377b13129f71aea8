"""Writes oracle_csa_tiny.npz: a regression snapshot of the oracle (calls only oracle/ and synth/)."""
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
import synth  # noqa: E402

SPEC = synth.LayerSpec(kind="csa", T=96, D=32, m=4, width=8, C=16, di=4, Hi=2, topk=6, window=8, H=2, dh=8,
                       scale=0.35, dtype="bf16", seed=11)


def compute():
    res = oracle.prefill(SPEC, synth.prefill_inputs(SPEC))
    return {"entries": res["entries"], "idx_keys": res["idx_keys"], "sel": res["sel"], "out": res["out"]}


if __name__ == "__main__":
    np.savez_compressed(os.path.join(HERE, "oracle_csa_tiny.npz"), **compute())
