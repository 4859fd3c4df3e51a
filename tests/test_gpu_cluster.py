"""Intra-block clustering selector against the oracle (needs a B200).

"AB-Attention: accurate block-sparse attention for video diffusion", TL;DR
fix (1): queries clustered within each query block; the block's score row is
the size-weighted mixture of its sub-centroids' rows.  k-means assignments are
decisions taken in floating point (fp32 on the GPU, fp64 in the oracle), so
near-equidistant tokens may land differently.  Blocks whose cluster sizes agree
(nearly all) must agree in centroids and score rows.  Every other block must be
a clustering that Lloyd's rounds reach when each token whose nearest centroids
are within 1e-4 (relative) of each other may take any of them: its sizes and
centroids must equal one of the end states of that branching replay.  Every
block's score row must equal the oracle's mixture fed the GPU's own
sub-centroids and sizes.
"""

import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_45_b200 import binding as bsa
from block_sparse_attention_45_b200 import synth
from tests import checkers

pytestmark = pytest.mark.gpu

CASES = {
    "tiny": synth.WORKLOADS["tiny"],
    "small": synth.WORKLOADS["small"],
    "h3_b2": synth.custom("h3_b2", batch=2, heads=3, head_dim=64, q_block=128, k_block=64,
                          text_len=100, num_frames=3, latent_h=10, latent_w=16, top_p=0.8,
                          seed=31),
    "h5_d128": synth.custom("h5_d128", heads=5, head_dim=128, q_block=64, k_block=128,
                            text_len=40, num_frames=3, latent_h=10, latent_w=10, top_p=0.7,
                            seed=32),
    # last query blocks of 5 and 3 tokens: fewer tokens than clusters (repeated seeds,
    # empty clusters of size 0)
    "tail5": synth.custom("tail5", heads=2, head_dim=64, q_block=64, k_block=64, text_len=69,
                          num_frames=2, latent_h=8, latent_w=8, top_p=0.8, seed=34),
    "tail3_d128": synth.custom("tail3_d128", heads=3, head_dim=128, q_block=128, k_block=128,
                               text_len=3, num_frames=2, latent_h=8, latent_w=16, top_p=0.8,
                               seed=35),
}

_CACHE = {}


def _inputs(name):
    if name not in _CACHE:
        w = CASES[name] if name in CASES else synth.WORKLOADS[name]
        _CACHE[name] = (w, synth.generate(w))
    return _CACHE[name]


def _dev_bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)


def _check_differing_block(x, n_sub, iters, c_g, s_g):
    for c, sizes in checkers.kmeans_end_states(x.astype(np.float64), n_sub, iters):
        if np.array_equal(sizes, s_g) and np.allclose(c_g, c, rtol=1e-4, atol=1e-4):
            return
    raise AssertionError("GPU clustering (sizes %s) is not reachable by the k-means rounds" %
                         s_g.tolist())


def _valid_tokens(w):
    cq = w.seq_pad // w.q_block
    return np.array([min(w.q_block, w.seq_len - i * w.q_block) for i in range(cq)])


@pytest.mark.parametrize("iters", [1, 3])
@pytest.mark.parametrize("n_sub", [1, 2, 4, 8, 16])
@pytest.mark.parametrize("name", sorted(CASES) + ["wan1.3b"])
def test_clustered_scores_match_the_oracle(name, n_sub, iters):
    if name == "wan1.3b" and (n_sub, iters) not in ((4, 3), (16, 1)):
        pytest.skip("full size: two configurations")
    w, x = _inputs(name)
    ora = oracle.default()
    L = w.layout()
    c_o, s_o = ora.subclusters(L, x["q"], n_sub, iters)
    kc_o = ora.pool(L, x["k"], w.k_block)
    p_o = ora.scores_clustered(L, c_o, s_o, kc_o)
    c_g, s_g, kc_g, p_g = bsa.block_scores_clustered(w, _dev_bf16(x["q"]), _dev_bf16(x["k"]), n_sub,
                                                     iters)
    torch.cuda.synchronize()
    c_g, s_g, p_g = c_g.cpu().numpy(), s_g.cpu().numpy(), p_g.cpu().numpy()
    np.testing.assert_allclose(kc_g.cpu().numpy(), kc_o, rtol=1e-5, atol=2e-6)
    # every block: sizes sum to its valid tokens, rows sum to one
    assert np.array_equal(s_g.sum(-1), np.broadcast_to(_valid_tokens(w), s_g.shape[:-1]))
    np.testing.assert_allclose(p_g.sum(-1), 1.0, atol=1e-5)
    same = (s_g == s_o).all(-1)
    assert same.mean() >= 0.99, same.mean()
    live = (s_o > 0)[same]
    np.testing.assert_allclose(c_g[same][live], c_o[same][live], rtol=1e-4, atol=1e-4)
    d = np.abs(p_g[same] - p_o[same])
    assert d.max() <= 1e-4, d.max()
    # every block's row: the oracle's mixture fed the GPU's own sub-centroids and sizes
    p_own = ora.scores_clustered(L, c_g, s_g, kc_o)
    d = np.abs(p_g - p_own)
    assert d.max() <= 1e-4, d.max()
    # blocks whose sizes differ: a clustering the rounds reach with near-ties taken either way
    cq = w.seq_pad // w.q_block
    xq = synth.bf16_bits_to_f32(x["q"]).reshape(w.batch * w.heads, w.seq_pad, w.head_dim)
    nvalid = _valid_tokens(w)
    for flat in np.nonzero(~same.reshape(-1))[0]:
        bh, i = flat // cq, flat % cq
        toks = xq[bh, i * w.q_block:i * w.q_block + nvalid[i]]
        _check_differing_block(toks, n_sub, iters, c_g.reshape(-1, n_sub, w.head_dim)[flat],
                               s_g.reshape(-1, n_sub)[flat])
    print("%s n_sub=%d iters=%d: %d blocks differ from the oracle's sizes, all reachable"
          % (name, n_sub, iters, int((~same).sum())))


@pytest.mark.parametrize("name", ["small", "h5_d128"])
def test_one_subcluster_is_the_block_centroid(name):
    w, x = _inputs(name)
    q, k = _dev_bf16(x["q"]), _dev_bf16(x["k"])
    c1, s1, _, p1 = bsa.block_scores_clustered(w, q, k, 1, 2)
    qc, _, p0 = bsa.block_scores(w, q, k)
    torch.cuda.synchronize()
    torch.testing.assert_close(c1[:, :, :, 0], qc, rtol=1e-6, atol=1e-6)
    assert torch.equal(s1[..., 0].cpu(), torch.from_numpy(_valid_tokens(w).astype(np.int32))
                       .expand_as(s1[..., 0].cpu()))
    torch.testing.assert_close(p1, p0, rtol=0, atol=2e-6)


def test_clustered_selection_end_to_end():
    """Clustered P' feeds the per-row top-p unchanged: the lists are the mask's
    compaction, every row keeps a top-p set of its own row."""
    w, x = _inputs("small")
    q, k = _dev_bf16(x["q"]), _dev_bf16(x["k"])
    _, _, _, p = bsa.block_scores_clustered(w, q, k, 4, 3)
    r = bsa.build_mask(w, p, [float(w.top_p)] * w.heads, 0)
    torch.cuda.synchronize()
    P = p.cpu().numpy().astype(np.float64)
    m = r["mask"].cpu().numpy().astype(bool)
    kept = np.where(m, P, 0).sum(-1)
    assert (kept >= np.float32(w.top_p) - 1e-5).all()
    # dropping the smallest kept entry falls short of p (shortest prefix)
    smallest = np.where(m, P, np.inf).min(-1)
    assert ((kept - smallest) < np.float32(w.top_p) + 1e-5).all()
