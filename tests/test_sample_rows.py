"""The full-size parity tests' choice of query blocks (CPU): it always ends, stays
inside the workload, holds every frame-0 block of the chosen head, and asks for
no more blocks than the workload has."""
import numpy as np
import pytest

import oracle
from block_sparse_attention_45_b200 import synth
from tests.gpu_util import sample_rows


@pytest.mark.parametrize("name", sorted(synth.WORKLOADS))
@pytest.mark.parametrize("kw", [dict(), dict(n_random=8, frame0_head=None), dict(n_random=2)])
def test_sample_rows_ends_and_covers(name, kw):
    w = synth.WORKLOADS[name]
    cq = w.seq_pad // w.q_block
    total = w.batch * w.heads * cq
    rows = sample_rows(w, **kw)
    assert len(np.unique(rows)) == len(rows) and rows.min() >= 0 and rows.max() < total
    assert len(rows) <= total
    if kw.get("frame0_head", 0) is not None:
        f0, f1 = oracle.frame0_qblocks(w.layout())
        assert set(range(f0, f1 + 1)) <= set(rows.tolist())
    n_random = kw.get("n_random", 64)
    if n_random >= w.batch * w.heads and total >= n_random + 4 + cq:
        # the random blocks go round every (batch, head) at least once
        assert set((rows // cq).tolist()) == set(range(w.batch * w.heads))
