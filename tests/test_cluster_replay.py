"""The k-means replay that judges GPU blocks whose clustering differs from the
oracle's ("AB-Attention ..." TL;DR fix (1), intra-block clusters): it must reach
the oracle's own clustering of every block, and reject one that no near-tie
explains (a token moved to a clearly farther cluster)."""
import numpy as np

import oracle
from block_sparse_attention_45_b200 import synth
from tests import checkers


def _blocks(w, x):
    xq = synth.bf16_bits_to_f32(x["q"]).reshape(w.batch * w.heads, w.seq_pad, w.head_dim)
    cq = w.seq_pad // w.q_block
    for bh in range(w.batch * w.heads):
        for i in range(cq):
            n = min(w.q_block, w.seq_len - i * w.q_block)
            yield bh * cq + i, xq[bh, i * w.q_block:i * w.q_block + n].astype(np.float64)


def _reached(states, c, s):
    return any(np.array_equal(sz, s) and np.allclose(cc, c, rtol=1e-4, atol=1e-4) for cc, sz in states)


def test_replay_reaches_the_oracle_clustering():
    w = synth.WORKLOADS["tiny"]
    x = synth.generate(w)
    ora = oracle.default()
    for n_sub, iters in ((2, 1), (4, 3), (16, 2)):
        c_o, s_o = ora.subclusters(w.layout(), x["q"], n_sub, iters)
        c_o = c_o.reshape(-1, n_sub, w.head_dim)
        s_o = s_o.reshape(-1, n_sub)
        for flat, toks in _blocks(w, x):
            states = checkers.kmeans_end_states(toks, n_sub, iters)
            assert _reached(states, c_o[flat], s_o[flat]), (n_sub, iters, flat)


def test_replay_rejects_a_moved_token():
    w = synth.WORKLOADS["tiny"]
    x = synth.generate(w)
    n_sub, iters = 4, 1
    _, toks = next(_blocks(w, x))
    states = checkers.kmeans_end_states(toks, n_sub, iters)
    assert len(states) == 1, "tiny block 0 has no near-tie"
    c, s = states[0]
    # reassign the token farthest from its own centroid's rivals to its second-nearest seed
    seeds = np.stack([toks[(k * len(toks)) // n_sub] for k in range(n_sub)])
    d = ((toks[:, None, :] - seeds[None]) ** 2).sum(-1)
    a = d.argmin(1)
    order = np.sort(d, 1)
    t = int(np.argmax(order[:, 1] - order[:, 0]))
    a[t] = int(np.argsort(d[t])[1])
    sizes = np.bincount(a, minlength=n_sub)
    moved = np.stack([toks[a == k].mean(0) if sizes[k] else seeds[k] for k in range(n_sub)])
    assert not _reached(states, moved, sizes)
