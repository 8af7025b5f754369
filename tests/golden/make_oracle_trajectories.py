"""Writes oracle_trajectories.json: the oracle's decode trajectories on the
tiny fp32 configuration (seed 0: 32 vision rows, 16 prompt and 16 committed
ids, block 4, 12 new tokens) for every decode driver, plus the fp8 decoder
model's threshold trajectory.  A regression record of the oracle, not a pin
to the pages: a later change of the oracle's arithmetic shows up as a
difference and must be regenerated with this script, its commit naming the
passage or reading that justifies it.

Usage: python tests/golden/make_oracle_trajectories.py
Calls only oracle/ and the input generator."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import dvlm_gen as gen  # noqa: E402
import oracle as O  # noqa: E402

OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_trajectories.json")
B, N_NEW = 4, 12


def trajectories() -> dict:
    d = O.dims_from(gen.TINY)
    w = O.weights_from_generator(gen, gen.TINY, 0)
    _, vis, ids = gen.decode_context(gen.TINY, 0, 32, 16, 16)
    vis = vis.astype(np.float64)

    def fresh(**kw):
        m = O.OracleModel(d, weights=w, bf16=False, Lmax=256, **kw)
        return m, O.prefill(m, vis, ids)

    out = {}
    m, s = fresh()
    out["threshold_tau0.9"] = O.decode_threshold(m, s, B, 0.9, N_NEW).tokens
    m, s = fresh()
    out["topk_k2"] = O.decode_threshold(m, s, B, 0.9, N_NEW, commit_k=2).tokens
    m, s = fresh()
    tr = O.decode_spec_linear(m, s, B, N_NEW)
    out["spec_linear"], out["spec_linear_accept"] = tr.tokens, tr.accept_lens
    m, s = fresh()
    tr = O.decode_spec_quadratic(m, s, B, N_NEW)
    out["spec_quadratic"], out["spec_quadratic_accept"] = tr.tokens, tr.accept_lens
    m, s = fresh()
    out["ar"] = O.decode_ar(m, s, N_NEW).tokens
    for k in (1, 2):
        m, s = fresh()
        tr = O.decode_lown(m, s, B, k, n_vis=32, max_new=N_NEW)
        out[f"routing_k{k}"] = tr.tokens
        out[f"routing_k{k}_passes"] = [tr.n_full, tr.n_text, tr.n_causal]
    m, s = fresh(fp8=True)
    out["fp8_threshold_tau0.9"] = O.decode_threshold(m, s, B, 0.9, N_NEW).tokens
    return {k: [int(v) for v in vals] for k, vals in out.items()}


if __name__ == "__main__":
    with open(OUT, "w") as f:
        json.dump(trajectories(), f, indent=1, sort_keys=True)
        f.write("\n")
    print(f"wrote {OUT}")
