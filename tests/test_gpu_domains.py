"""Pooled top-p over the competition domains against the oracle (needs a B200).

"Competition Domains Matter ..." s3: the pairs (h, i, j) of a batch entry
compete per row, per head, per entropy group (both halves pooled), across all
heads, or as EG-Sparse (the low-entropy half pooled, the rest per row).  On the
oracle's P' and value norms the GPU's pools must equal the oracle's routing
(exactly where the routing does not depend on the entropies, and wherever the
two heads around the median are apart where it does), and its masks the
oracle's pooled selection on that routing.
"""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_45_b200 import binding as bsa
from block_sparse_attention_45_b200 import synth
from tests import checkers
from tests.test_gpu_eg import CASES, _dev_bf16, _median_gap, _oracle_inputs

pytestmark = pytest.mark.gpu

DOMAINS = {"row": bsa.DOMAIN_ROW, "head": bsa.DOMAIN_HEAD, "grouped": bsa.DOMAIN_GROUPED,
           "all": bsa.DOMAIN_ALL, "eg": bsa.DOMAIN_EG}
ENTROPY_ROUTED = (bsa.DOMAIN_GROUPED, bsa.DOMAIN_EG)


def _routed_alike(w, H, gpu_pool, ora_pool, domain):
    """Per batch entry: whether the GPU's pools equal the oracle's; asserts it
    where the routing is decided by more than the entropies' rounding."""
    gap = _median_gap(H)
    same = []
    for b in range(w.batch):
        eq = bool(np.array_equal(gpu_pool[b], ora_pool[b]))
        if domain not in ENTROPY_ROUTED or gap[b] > 1e-4 * max(1.0, float(np.abs(H[b]).max())):
            assert eq, (b, domain, gpu_pool[b], ora_pool[b], H[b])
        same.append(eq)
    return same


@pytest.mark.parametrize("value_aware", [True, False], ids=["value_aware", "pprime"])
@pytest.mark.parametrize("pool_p", [0.9, 0.5, 0.0, 1.5])
@pytest.mark.parametrize("dname", sorted(DOMAINS))
@pytest.mark.parametrize("name", sorted(CASES))
def test_domain_on_oracle_inputs(name, dname, pool_p, value_aware):
    domain = DOMAINS[dname]
    w, _, probs, H, vn = _oracle_inputs(name)
    ora = oracle.default()
    L = w.layout()
    tp = [float(w.top_p)] * w.heads
    vn_used = vn if value_aware else None
    g = bsa.build_mask_domain(w, domain, torch.from_numpy(probs).cuda(),
                              None if vn_used is None else torch.from_numpy(vn_used).cuda(),
                              tp, pool_p, 0)
    torch.cuda.synchronize()
    np.testing.assert_allclose(g["entropy"].cpu().numpy(), H, rtol=checkers.ENTROPY_REL)
    pool_o, G = ora.domain_route(L, H, domain)
    pool_g = g["pool_of"].cpu().numpy()
    same = _routed_alike(w, H, pool_g, pool_o, domain)
    exp = ora.pool_select(L, probs, vn_used, tp, pool_p, pool_o, G)
    got = g["mask"].cpu().numpy()
    for b in range(w.batch):
        if same[b]:
            bad = np.argwhere((got[b] != exp[b]).any(-1))
            assert bad.size == 0, (name, dname, pool_p, b, bad[:5].tolist())
    checkers.check_lists(g["kv_index"].cpu().numpy(), g["kv_count"].cpu().numpy(), got)
    pooled = pool_g >= 0
    if pool_p <= 0:   # a pooled row keeps exactly its best block
        assert (got[pooled].sum(-1) == 1).all()
    if pool_p > 1:    # everything pooled is kept
        assert got[pooled].all()


@pytest.mark.parametrize("name", ["small", "h3_b2", "h5_d128"])
def test_eg_domain_is_build_mask_eg(name):
    w, _, probs, _, vn = _oracle_inputs(name)
    tp = [float(w.top_p)] * w.heads
    p, v = torch.from_numpy(probs).cuda(), torch.from_numpy(vn).cuda()
    d = bsa.build_mask_domain(w, bsa.DOMAIN_EG, p, v, tp, 0.9, w.flags)
    e = bsa.build_mask_eg(w, p, v, tp, 0.9, w.flags)
    torch.cuda.synchronize()
    for key in ("mask", "kv_count", "entropy"):
        assert torch.equal(d[key], e[key]), key
    # list entries past kv_count are unspecified
    valid = torch.arange(d["kv_index"].shape[-1], device=d["kv_index"].device) < d["kv_count"][..., None]
    assert torch.equal(torch.where(valid, d["kv_index"], -1), torch.where(valid, e["kv_index"], -1))
    assert torch.equal((d["pool_of"] >= 0).to(torch.uint8), e["low_heads"])


@pytest.mark.parametrize("name", ["small", "h3_b2"])
def test_row_domain_is_build_mask(name):
    w, _, probs, _, _ = _oracle_inputs(name)
    tp = [float(w.top_p)] * w.heads
    p = torch.from_numpy(probs).cuda()
    d = bsa.build_mask_domain(w, bsa.DOMAIN_ROW, p, None, tp, 0.9, w.flags)
    r = bsa.build_mask(w, p, tp, w.flags)
    torch.cuda.synchronize()
    assert (d["pool_of"] == -1).all()
    assert torch.equal(d["mask"], r["mask"]) and torch.equal(d["kv_count"], r["kv_count"])


@pytest.mark.parametrize("dname", ["head", "grouped", "all"])
@pytest.mark.parametrize("name", ["h3_b2", "h5_d128"])
def test_domain_many_ties(name, dname):
    """Quantised scores (powers of two): the cut of each pool falls inside a run of
    equal scores spread over many rows and heads."""
    domain = DOMAINS[dname]
    w = CASES[name]
    ora = oracle.default()
    L = w.layout()
    B, H = w.batch, w.heads
    Cq, Ck = w.seq_pad // w.q_block, w.seq_pad // w.k_block
    rng = np.random.default_rng(11)
    probs = (2.0 ** -rng.integers(3, 7, size=(B, H, Cq, Ck))).astype(np.float32)
    vn = (2.0 ** rng.integers(0, 2, size=(B, H, Ck))).astype(np.float32)
    tp = [0.8] * H
    H_ora, _ = ora.entropy(L, probs)
    for pool_p in (0.5, 0.9):
        g = bsa.build_mask_domain(w, domain, torch.from_numpy(probs).cuda(), torch.from_numpy(vn).cuda(),
                                  tp, pool_p, 0)
        torch.cuda.synchronize()
        pool_o, G = ora.domain_route(L, H_ora, domain)
        pool_g = g["pool_of"].cpu().numpy()
        exp = ora.pool_select(L, probs, vn, tp, pool_p, pool_o, G)
        got = g["mask"].cpu().numpy()
        for b in range(B):
            if np.array_equal(pool_g[b], pool_o[b]):
                bad = np.argwhere((got[b] != exp[b]).any(-1))
                assert bad.size == 0, (name, dname, pool_p, b, bad[:5].tolist())
        checkers.check_lists(g["kv_index"].cpu().numpy(), g["kv_count"].cpu().numpy(), got)


@pytest.mark.parametrize("dname", ["head", "grouped", "all"])
def test_domain_full_size_against_the_oracle(dname):
    """Wan2.1-1.3B at full size (12 heads, 32,760 tokens, C = 256) on the GPU's own P'
    and value norms: the masks equal the oracle's pooled selection on the same scores."""
    domain = DOMAINS[dname]
    w = synth.WORKLOADS["wan1.3b"]
    x = synth.generate(w)
    q, k, v = _dev_bf16(x["q"]), _dev_bf16(x["k"]), _dev_bf16(x["v"])
    _, _, probs = bsa.block_scores(w, q, k)
    vn = bsa.value_norms(w, v)
    tp = [0.9] * w.heads
    g = bsa.build_mask_domain(w, domain, probs, vn, tp, 0.9, 0)
    torch.cuda.synchronize()
    ora = oracle.default()
    L = w.layout()
    P, V = probs.cpu().numpy(), vn.cpu().numpy()
    pool_g = g["pool_of"].cpu().numpy()
    if domain == bsa.DOMAIN_GROUPED:   # route by the GPU's split (its own entropies)
        G = 2
        pool_o = pool_g
        assert ((pool_g == 0).sum(-1) == w.heads // 2).all()
    else:
        H_ora, _ = ora.entropy(L, P)
        pool_o, G = ora.domain_route(L, H_ora, domain)
        assert np.array_equal(pool_g, pool_o)
    exp = ora.pool_select(L, P, V, tp, 0.9, pool_o, G)
    got = g["mask"].cpu().numpy()
    bad = np.argwhere((got != exp).any(-1))
    assert bad.size == 0, bad[:5].tolist()
    checkers.check_lists(g["kv_index"].cpu().numpy(), g["kv_count"].cpu().numpy(), got)
