"""Write tests/golden/digests.json: SHA-256 digests of oracle outputs.

The paper "DeepSeek-V4-Flash on AMD gfx90a: Correctness Recovery and
Inference Performance Engineering" (abstract) fixed its W2 layout bug with
fixed-token and hash-based checks before optimising further.  These digests
play that role here.  Every value comes from the oracle (oracle/) fed by the
seeded input generator (synth/); nothing here touches the CUDA library.

Usage: python tests/golden/make_golden.py [workload ...]
(with names, only those entries are recomputed; the others are kept)
"""
import hashlib
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import synth  # noqa: E402

OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "digests.json")
FULL = ["tiny_T4", "decode_T8", "decode_T64"]        # whole layer
SAMPLED = ["prefill_T4604", "prefill_skew_T16384",     # route/sort whole, layer on sampled tokens
           "prefill_skew1.25_T16384"]


def sha(a: np.ndarray) -> str:
    return hashlib.sha256(np.ascontiguousarray(a).tobytes()).hexdigest()


def sample_tokens(T: int):
    return sorted({0, 1, T // 3, T // 2, T - 2, T - 1})


def digests(name: str) -> dict:
    w = synth.WORKLOADS[name]
    d = synth.make(w)
    out = {"x": sha(d["x"]), "logits": sha(d["logits"])}
    if name in FULL:
        o = oracle.forward(d["x"], d["logits"], d["w1_codes"], d["w1_scales"], d["w2_codes"],
                           d["w2_scales"], w.k)
        for key in ["idx", "gates", "counts", "offsets", "perm", "pos", "xq", "sx", "hq", "sh", "y"]:
            out[key] = sha(o[key])
    else:
        idx, gates = oracle.route(d["logits"], w.k)
        counts, offsets, perm, pos = oracle.sort(idx, w.E)
        for key, v in dict(idx=idx, gates=gates, counts=counts, offsets=offsets, perm=perm,
                           pos=pos).items():
            out[key] = sha(v)
        tok = sample_tokens(w.T)
        ot = oracle.forward_tokens(d["x"], d["logits"], d["w1_codes"], d["w1_scales"],
                                   d["w2_codes"], d["w2_scales"], w.k, tok)
        out["sample_tokens"] = tok
        for key in ["xq", "sx", "hq", "sh", "y"]:
            out["sample_" + key] = sha(ot[key])
        out["touched_experts"] = int((counts > 0).sum())
        out["max_rows_per_expert"] = int(counts.max())
    return out


def main():
    names = sys.argv[1:] or FULL + SAMPLED
    res = json.load(open(OUT)) if sys.argv[1:] and os.path.exists(OUT) else {}
    for name in names:
        res[name] = digests(name)
        print(name, "done", flush=True)
    with open(OUT, "w") as f:
        json.dump(res, f, indent=1, sort_keys=True)


if __name__ == "__main__":
    main()
