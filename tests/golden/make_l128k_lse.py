"""Write the complete fp64 LSE of heads 0 and 1 of the causal 128K workload.

Workload: B=1, Hq=Hkv=32, L=131072, d=128, eight ring blocks of 16384 rows,
causal, scale 1/sqrt(128), inputs from ``inputs.workload_inputs`` (seed 3).
The file ``l128k_h32_causal_lse_h01.npy`` holds lse[0, h, r] for h in {0, 1}
and every row r, float64 [2, 131072], natural log, as computed by the fp64
oracle (``oracle.attention_rows``: the plain definition, row by row).  The
companion ``l128k_h32_causal_lse_h01.json`` records the workload, the SHA-256
of the bf16 inputs of those two heads, so a test can tell a changed input
generator from a wrong kernel, and the SHA-256 of the array.

Only ``oracle/`` computes anything here.  Run from the repository root:
``python tests/golden/make_l128k_lse.py`` (about 10 minutes on 8 cores).
"""

from __future__ import annotations

import hashlib
import json
import os
import sys
import time

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)
sys.path.insert(0, os.path.dirname(HERE))

NAME = "l128k_h32_causal_lse_h01"
HEADS = (0, 1)


def input_digest(q, k, v, heads):
    """SHA-256 over the bf16 bits of q[:, :, h], k[:, :, h // g], v[:, :, h // g]."""
    import torch
    g = q.shape[2] // k.shape[2]
    h = hashlib.sha256()
    for hd in heads:
        for t, i in ((q, hd), (k, hd // g), (v, hd // g)):
            h.update(t[:, :, i].contiguous().view(torch.int16).numpy().tobytes())
    return h.hexdigest()


def main():
    import numpy as np

    from oracle_pool import attention_rows_parallel
    from ring_attention_ordered_b200.inputs import WORKLOADS, workload_inputs

    w = WORKLOADS["l128k_h32_causal"]
    t0 = time.time()
    q, k, v = workload_inputs(w)
    g = w.group
    kvh = sorted({h // g for h in HEADS})
    # keep only the heads the file covers (the oracle sees a 2-head problem
    # with the same per-head data and the same grouping)
    qs = q[:, :, list(HEADS)].contiguous()
    ks = k[:, :, kvh].contiguous()
    vs = v[:, :, kvh].contiguous()
    assert qs.shape[2] // ks.shape[2] == 1 or g == len(HEADS) // len(kvh)
    digest = input_digest(q, k, v, HEADS)
    del q, k, v
    rows = np.arange(w.L, dtype=np.int64)
    bhr = np.concatenate([np.stack([np.zeros_like(rows), np.full_like(rows, i), rows], axis=1)
                          for i in range(len(HEADS))])
    _, lse = attention_rows_parallel(qs, ks, vs, w.causal, w.scale, bhr)
    lse = lse.reshape(len(HEADS), w.L)
    path = os.path.join(HERE, NAME + ".npy")
    np.save(path, lse)
    meta = {
        "workload": w.name, "describe": w.describe(), "seed": w.seed, "heads": list(HEADS),
        "rows": w.L, "dtype": "float64", "what": "lse[0, h, :] natural log, fp64 oracle",
        "inputs_sha256": digest,
        "array_sha256": hashlib.sha256(lse.tobytes()).hexdigest(),
        "script": "tests/golden/make_l128k_lse.py", "seconds": round(time.time() - t0, 1),
    }
    with open(os.path.join(HERE, NAME + ".json"), "w") as f:
        json.dump(meta, f, indent=1)
        f.write("\n")
    print(json.dumps(meta))


if __name__ == "__main__":
    main()
