"""The stored complete LSE of heads 0 and 1 of the causal 128K workload
(tests/golden/make_l128k_lse.py) and the parallel oracle runner it uses,
checked on the CPU: the runner equals ``oracle.attention_rows``; the stored
file is intact, was made from the inputs the generator draws now, has the
closed form at row 0 (one key: lse = scale q_0 . k_0) and agrees with the
oracle re-run on sampled rows."""

from __future__ import annotations

import hashlib
import json
import os

import numpy as np
import torch

import oracle
from oracle_pool import attention_rows_parallel, split_by_work


def test_pool_equals_the_oracle():
    from ring_attention_ordered_b200.inputs import make_inputs
    q, k, v = make_inputs(2, 4, 2, 300, 64, seed=21)
    bhr = np.array([[b, h, r] for b in range(2) for h in range(4) for r in range(300)])
    bhr = bhr[np.random.default_rng(1).permutation(len(bhr))]
    for causal in (True, False):
        o1, l1 = oracle.attention_rows(q, k, v, causal, 0.125, bhr)
        o2, l2 = attention_rows_parallel(q, k, v, causal, 0.125, bhr, workers=2)
        np.testing.assert_allclose(o2, o1, rtol=0, atol=1e-13)
        np.testing.assert_allclose(l2, l1, rtol=0, atol=1e-13)


def test_split_by_work_covers_every_row_once():
    bhr = np.array([[0, 0, r] for r in range(1000)])
    parts = split_by_work(bhr, 1000, True, 7)
    assert np.array_equal(np.sort(np.concatenate(parts)), np.arange(1000))
    work = [float((bhr[p, 2] + 1).sum()) for p in parts]
    assert max(work) < 1.3 * (sum(work) / len(work))


def test_stored_l128k_lse(golden_dir):
    from ring_attention_ordered_b200.inputs import WORKLOADS, workload_inputs
    w = WORKLOADS["l128k_h32_causal"]
    meta = json.load(open(os.path.join(golden_dir, "l128k_h32_causal_lse_h01.json")))
    lse = np.load(os.path.join(golden_dir, "l128k_h32_causal_lse_h01.npy"))
    assert meta["workload"] == w.name and lse.shape == (len(meta["heads"]), w.L)
    assert hashlib.sha256(lse.tobytes()).hexdigest() == meta["array_sha256"]
    q, k, v = workload_inputs(w)
    digest = hashlib.sha256()
    for hd in meta["heads"]:
        for t, i in ((q, hd), (k, hd // w.group), (v, hd // w.group)):
            digest.update(t[:, :, i].contiguous().view(torch.int16).numpy().tobytes())
    assert digest.hexdigest() == meta["inputs_sha256"]
    for i, hd in enumerate(meta["heads"]):
        row0 = w.scale * float((q[0, 0, hd].double() * k[0, 0, hd // w.group].double()).sum())
        assert abs(lse[i, 0] - row0) < 1e-12
    rng = np.random.default_rng(7)
    bhr = np.array([[0, meta["heads"][i % 2], r] for i, r in
                    enumerate(rng.choice(w.L, size=6, replace=False))] +
                   [[0, meta["heads"][1], w.L - 1]])
    _, ref = oracle.attention_rows(q, k, v, True, w.scale, bhr)
    got = lse[[meta["heads"].index(h) for h in bhr[:, 1]], bhr[:, 2]]
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-10)
