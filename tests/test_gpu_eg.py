"""Entropy-guided grouped cross-head selection against the oracle (needs a B200).

"Competition Domains Matter ..." s3.3 domain 3 (heads split at the median of
their entropy; the low-entropy heads compete in one pool per batch entry), the
one-key-per-row safeguard, and s4 (the pool ranks pairs by P' * ||c^V||).
On identical inputs (the oracle's P' and value norms) the GPU routing and masks
must equal the oracle's; on the GPU's own inputs the result must satisfy the
rule's defining properties.
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
    "tiny": synth.WORKLOADS["tiny"],                                     # H = 2: one pooled head
    "small": synth.WORKLOADS["small"],
    "h3_b2": synth.custom("h3_b2", batch=2, heads=3, head_dim=64, q_block=128, k_block=64,
                          text_len=100, num_frames=3, latent_h=10, latent_w=16, top_p=0.8,
                          seed=31),                                      # odd H, two batch entries
    "h5_d128": synth.custom("h5_d128", heads=5, head_dim=128, q_block=64, k_block=128,
                            text_len=40, num_frames=3, latent_h=10, latent_w=10, top_p=0.7,
                            seed=32),
    "h1": synth.custom("h1", heads=1, head_dim=64, q_block=128, k_block=128, text_len=20,
                       num_frames=3, latent_h=10, latent_w=16, top_p=0.85, seed=33),
}

_CACHE = {}


def _oracle_inputs(name):
    if name not in _CACHE:
        w = CASES[name]
        x = synth.generate(w)
        ora = oracle.default()
        L = w.layout()
        qc = ora.pool(L, x["q"], w.q_block)
        kc = ora.pool(L, x["k"], w.k_block)
        probs = ora.scores(L, qc, kc)
        H, _ = ora.entropy(L, probs)
        vn = ora.value_norms(L, x["v"])
        _CACHE[name] = (w, x, probs, H, vn)
    return _CACHE[name]


def _dev_bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)


@pytest.mark.parametrize("name", sorted(CASES))
def test_value_norms(name):
    w, x, _, _, vn = _oracle_inputs(name)
    got = bsa.value_norms(w, _dev_bf16(x["v"]))
    torch.cuda.synchronize()
    np.testing.assert_allclose(got.cpu().numpy(), vn, rtol=1e-5, atol=1e-6)


def _median_gap(H):
    """Per batch entry: the entropy gap between the last pooled and the first
    per-row head in (H asc) order (inf when nothing is pooled)."""
    gaps = []
    for row in np.asarray(H, np.float64):
        s = np.sort(row)
        k = len(s) // 2
        gaps.append(np.inf if k == 0 else s[k] - s[k - 1])
    return np.array(gaps)


@pytest.mark.parametrize("value_aware", [True, False], ids=["value_aware", "pprime"])
@pytest.mark.parametrize("pool_p", [0.9, 0.5, 0.0, 1.5])
@pytest.mark.parametrize("name", sorted(CASES))
def test_eg_on_oracle_inputs(name, pool_p, value_aware):
    w, _, probs, H, vn = _oracle_inputs(name)
    ora = oracle.default()
    L = w.layout()
    tp = [float(w.top_p)] * w.heads
    vn_used = vn if value_aware else None
    g = bsa.build_mask_eg(w, torch.from_numpy(probs).cuda(),
                          None if vn_used is None else torch.from_numpy(vn_used).cuda(),
                          tp, pool_p, 0)
    torch.cuda.synchronize()
    np.testing.assert_allclose(g["entropy"].cpu().numpy(), H, rtol=checkers.ENTROPY_REL)
    low = ora.eg_route(L, H)
    gpu_low = g["low_heads"].cpu().numpy()
    assert np.array_equal(gpu_low.sum(-1), np.full(w.batch, w.heads // 2))
    # the routing must match wherever the two heads around the median are apart
    gap = _median_gap(H)
    same = [bool(np.array_equal(gpu_low[b], low[b])) for b in range(w.batch)]
    for b in range(w.batch):
        if gap[b] > 1e-4 * max(1.0, float(np.abs(H[b]).max())):
            assert same[b], (b, gpu_low[b], low[b], H[b])
    # masks on the oracle's own routing, for the batch entries routed alike
    exp = ora.eg_select(L, probs, vn_used, tp, pool_p, low)
    got = g["mask"].cpu().numpy()
    for b in range(w.batch):
        if same[b]:
            bad = np.argwhere((got[b] != exp[b]).any(-1))
            assert bad.size == 0, (name, pool_p, b, bad[:5].tolist())
    checkers.check_lists(g["kv_index"].cpu().numpy(), g["kv_count"].cpu().numpy(), got)
    if pool_p <= 0:   # a pooled row keeps exactly its best block
        assert (got[gpu_low.astype(bool)].sum(-1) == 1).all()
    if pool_p > 1:    # everything pooled is kept
        assert got[gpu_low.astype(bool)].all()


@pytest.mark.parametrize("name", ["small", "h3_b2"])
def test_eg_overrides_and_per_row_heads(name):
    w, _, probs, H, vn = _oracle_inputs(name)
    ora = oracle.default()
    L = w.layout()
    tp = [float(w.top_p)] * w.heads
    g = bsa.build_mask_eg(w, torch.from_numpy(probs).cuda(), torch.from_numpy(vn).cuda(), tp,
                          0.9, w.flags)
    g0 = bsa.build_mask(w, torch.from_numpy(probs).cuda(), tp, 0)
    torch.cuda.synchronize()
    low = g["low_heads"].cpu().numpy()
    exp = ora.overrides(L, w.flags, ora.eg_select(L, probs, vn, tp, 0.9, low))
    assert np.array_equal(g["mask"].cpu().numpy(), exp)
    # per-row heads take exactly the per-row rule of bsa_build_mask
    per_row = ~low.astype(bool)
    m0 = ora.overrides(L, w.flags, g0["mask"].cpu().numpy())
    assert np.array_equal(g["mask"].cpu().numpy()[per_row], m0[per_row])


@pytest.mark.parametrize("kind", ["uniform", "quantised"])
@pytest.mark.parametrize("name", ["h3_b2", "h5_d128", "small"])
def test_eg_many_ties(name, kind):
    """Scores with many exact ties: the cut falls inside a run of equal scores
    spread over many rows, so the kept ties follow the (h, i, j) order."""
    w = CASES[name]
    ora = oracle.default()
    L = w.layout()
    B, H = w.batch, w.heads
    Cq, Ck = w.seq_pad // w.q_block, w.seq_pad // w.k_block
    rng = np.random.default_rng(7)
    if kind == "uniform":
        probs = np.full((B, H, Cq, Ck), 1.0 / Ck, np.float32)
        vn = np.ones((B, H, Ck), np.float32)
        # distinct per-head entropies would all be equal here: the routing then
        # follows the head index
    else:
        probs = (2.0 ** -rng.integers(3, 7, size=(B, H, Cq, Ck))).astype(np.float32)
        vn = (2.0 ** rng.integers(0, 2, size=(B, H, Ck))).astype(np.float32)
    tp = [0.8] * H
    H_ora, _ = ora.entropy(L, probs)
    for pool_p in (0.5, 0.9, 0.0):
        g = bsa.build_mask_eg(w, torch.from_numpy(probs).cuda(), torch.from_numpy(vn).cuda(), tp,
                              pool_p, 0)
        torch.cuda.synchronize()
        gpu_low = g["low_heads"].cpu().numpy()
        low = ora.eg_route(L, H_ora)
        exp = ora.eg_select(L, probs, vn, tp, pool_p, low)
        got = g["mask"].cpu().numpy()
        for b in range(B):
            if np.array_equal(gpu_low[b], low[b]):
                bad = np.argwhere((got[b] != exp[b]).any(-1))
                assert bad.size == 0, (name, kind, pool_p, b, bad[:5].tolist())
        checkers.check_lists(g["kv_index"].cpu().numpy(), g["kv_count"].cpu().numpy(), got)


def test_eg_zero_eps_routes_every_batch_entry():
    """eps = 0 (entropy terms of zero entries are 0 * log 0): the median split
    still pools exactly floor(H/2) heads per batch entry."""
    w, _, probs, _, vn = _oracle_inputs("h3_b2")
    p = probs.copy()
    p[..., ::3] = 0.0
    g = bsa.build_mask_eg(w, torch.from_numpy(p).cuda(), torch.from_numpy(vn).cuda(),
                          [0.8] * w.heads, 0.9, 0, eps=0.0)
    torch.cuda.synchronize()
    low = g["low_heads"].cpu().numpy()
    assert np.array_equal(low.sum(-1), np.full(w.batch, w.heads // 2))
    checkers.check_lists(g["kv_index"].cpu().numpy(), g["kv_count"].cpu().numpy(),
                         g["mask"].cpu().numpy())


@pytest.mark.parametrize("name", ["small", "h3_b2", "h5_d128"])
def test_eg_centroid_distortion(name):
    """The competition-domain diagnostic ("Competition Domains Matter ..." s3: relative
    Frobenius error of the masked, row-renormalised centroid output): the GPU's masks
    give the oracle's distortion per head, every value in [0, 1), and keeping every block
    gives zero (up to the fp32 rows' rounding)."""
    w, x, probs, H, vn = _oracle_inputs(name)
    ora = oracle.default()
    L = w.layout()
    vcent = ora.pool(L, x["v"], w.k_block)
    tp = [float(w.top_p)] * w.heads
    g = bsa.build_mask_eg(w, torch.from_numpy(probs).cuda(), torch.from_numpy(vn).cuda(), tp, 0.9, 0)
    r = bsa.build_mask(w, torch.from_numpy(probs).cuda(), tp, 0)
    torch.cuda.synchronize()
    low = ora.eg_route(L, H)
    e_gpu = ora.centroid_distortion(L, probs, vcent, g["mask"].cpu().numpy())
    e_ora = ora.centroid_distortion(L, probs, vcent, ora.eg_select(L, probs, vn, tp, 0.9, low))
    same = (g["low_heads"].cpu().numpy() == low).all(-1)
    np.testing.assert_allclose(e_gpu[same], e_ora[same], rtol=1e-12, atol=1e-15)
    e_row = ora.centroid_distortion(L, probs, vcent, r["mask"].cpu().numpy())
    assert ((e_gpu >= 0) & (e_gpu < 1)).all() and ((e_row >= 0) & (e_row < 1)).all()
    full = np.ones_like(probs, dtype=np.uint8)   # zero up to the fp32 rows' sum (1 +- 1e-7)
    assert (ora.centroid_distortion(L, probs, vcent, full) < 1e-6).all()


def test_eg_single_head_is_the_per_row_rule():
    w, _, probs, _, vn = _oracle_inputs("h1")
    tp = [float(w.top_p)]
    g = bsa.build_mask_eg(w, torch.from_numpy(probs).cuda(), torch.from_numpy(vn).cuda(), tp, 0.3,
                          w.flags)
    r = bsa.build_mask(w, torch.from_numpy(probs).cuda(), tp, w.flags)
    torch.cuda.synchronize()
    assert int(g["low_heads"].sum().item()) == 0
    assert torch.equal(g["mask"], r["mask"]) and torch.equal(g["kv_count"], r["kv_count"])


@pytest.mark.parametrize("wname", ["wan1.3b", "wan14b"])
def test_eg_full_pipeline_properties(wname):
    """GPU P' and value norms at full size (Wan2.1-1.3B: 12 heads; Wan2.1-14B: 40 heads,
    64-key blocks): the pooled selection is the shortest prefix reaching pool_p of the
    pool (checked on the GPU's own scores), every pooled row is non-empty, and the lists
    match the mask."""
    w = synth.WORKLOADS[wname]
    x = synth.generate(w)
    q, k, v = _dev_bf16(x["q"]), _dev_bf16(x["k"]), _dev_bf16(x["v"])
    _, _, probs = bsa.block_scores(w, q, k)
    vn = bsa.value_norms(w, v)
    tp = [0.9] * w.heads
    pool_p = 0.9
    g = bsa.build_mask_eg(w, probs, vn, tp, pool_p, 0)
    torch.cuda.synchronize()
    m = g["mask"].cpu().numpy().astype(bool)
    low = g["low_heads"].cpu().numpy().astype(bool)
    checkers.check_lists(g["kv_index"].cpu().numpy(), g["kv_count"].cpu().numpy(), m)
    P = probs.cpu().numpy()
    V = vn.cpu().numpy()
    for b in range(w.batch):
        hs = np.nonzero(low[b])[0]
        assert len(hs) == w.heads // 2
        I = (P[b, hs] * V[b, hs][:, None, :]).astype(np.float32)   # the fp32 scores
        kept = m[b, hs]
        assert kept.any(-1).all()                                  # the safeguard
        target = pool_p * I.astype(np.float64).sum()
        tau = I[~kept].max()                                       # best pair left out
        assert kept[I > tau].all()                                 # everything above it is kept
        prefix = I[kept & (I >= tau)].astype(np.float64)           # the pool's prefix
        assert prefix.sum() >= target * (1 - 1e-6)                 # reaches the target
        assert prefix.sum() - prefix.min() < target * (1 + 1e-6)   # and is the shortest
    # per-row heads: the per-row rule of bsa_build_mask on the same P'
    r = bsa.build_mask(w, probs, tp, 0)
    torch.cuda.synchronize()
    assert np.array_equal(m[~low], r["mask"].cpu().numpy().astype(bool)[~low])
