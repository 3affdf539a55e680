"""Write tiny_decode_oracle.json: the float64 oracle on the seeded tiny decode batch.

Calls only oracle/ (inputs from the seeded generator). Run from the repository root:
    python tests/golden/make_golden.py
"""
import hashlib
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import workloads as W  # noqa: E402


def compute():
    b = W.make_config("tiny_decode")
    qs, ks, vs = [], [], []
    for i in range(len(b.seqs)):
        k, v = b.seq_kv(i)
        qs.append(b.seq_q(i).double().numpy())
        ks.append(k.double().numpy())
        vs.append(v.double().numpy())
    out = oracle.attention(qs, ks, vs, b.query_lens, b.mask_kinds, [s.parents for s in b.seqs])
    h = hashlib.sha256()
    for t in (b.q, b.k, b.v):
        h.update(t.view(dtype=__import__("torch").int16).numpy().tobytes())
    return out, h.hexdigest()


if __name__ == "__main__":
    out, digest = compute()
    rec = {"what": "float64 oracle output on the seeded tiny decode batch",
           "inputs_sha256": digest, "shape": list(out.shape),
           "rows": np.round(out.reshape(out.shape[0], -1), 12).tolist()}
    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_decode_oracle.json"), "w") as f:
        json.dump(rec, f)
    print("wrote", out.shape, digest)
