"""Dynamic Head Programming through the C ABI's host entry point (no GPU).

"Efficient Autoregressive Video Diffusion with Dummy Head", Step 1: the page's
worked example, agreement with the oracle on random frame scores, and
argument validation.
"""
import json
import os

import numpy as np

import oracle
from block_sparse_attention_45_b200 import binding as bsa

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_worked_example():
    g = json.load(open(os.path.join(GOLDEN, "dhp_example.json")))
    a = np.zeros((g["heads"], 3), np.float32)
    for h, x in enumerate(g["l"]):
        a[h, h % 2] = x
        a[h, 1 - h % 2] = x / 3
        a[h, 2] = 1 - x - x / 3
    lab = bsa.dhp_labels(a, g["n_dummy"])
    assert sorted(np.nonzero(lab == bsa.HEAD_DUMMY)[0].tolist()) == g["dummy_heads"]
    assert [int(lab[h]) for h in range(8) if lab[h] != bsa.HEAD_DUMMY] == [0, 1, 0, 1]
    ex = np.array([e["alpha"] for e in g["step0_examples"]], np.float32)
    assert bsa.dhp_labels(ex, 1).tolist() == [bsa.HEAD_NEIGHBOR, bsa.HEAD_DUMMY]


def test_matches_the_oracle():
    ora = oracle.default()
    rng = np.random.default_rng(3)
    for H in (1, 5, 12, 40):
        for _ in range(20):
            a = rng.dirichlet([1.0, 1.0, 1.0], size=H).astype(np.float32)
            a[rng.random(H) < 0.2, 0] = a[0, 1]       # some exact ties in l and between roles
            for n in (0, H // 2, H):
                assert np.array_equal(bsa.dhp_labels(a, n), ora.dhp(a.astype(np.float64), n))


def test_validation():
    import ctypes
    lib = bsa.load()
    a = np.zeros((4, 3), np.float32)
    lab = np.zeros(4, np.int32)
    pa, pl = a.ctypes.data_as(ctypes.c_void_p), lab.ctypes.data_as(ctypes.c_void_p)
    assert lib.bsa_dhp_labels(None, 4, 1, pl) == bsa.BSA_ERR_INVALID_ARG
    assert lib.bsa_dhp_labels(pa, 4, 1, None) == bsa.BSA_ERR_INVALID_ARG
    assert lib.bsa_dhp_labels(pa, 0, 0, pl) == bsa.BSA_ERR_INVALID_ARG
    assert lib.bsa_dhp_labels(pa, 4, 5, pl) == bsa.BSA_ERR_INVALID_ARG
    assert lib.bsa_dhp_labels(pa, 4, -1, pl) == bsa.BSA_ERR_INVALID_ARG
    a[2, 1] = np.nan
    assert lib.bsa_dhp_labels(pa, 4, 1, pl) == bsa.BSA_ERR_INVALID_ARG
