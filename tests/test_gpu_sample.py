"""Importance sampling with inverse-inclusion-probability weights against the
oracle (needs a B200).

"AB-Attention: accurate block-sparse attention for video diffusion", TL;DR
fix (2): blocks sampled in proportion to importance and reweighted by the
inverse inclusion probability, so one pass estimates dense attention without
bias.  The draw is a function of (seed, pair index), so the GPU's samples,
lists and weights must equal the oracle's bit for bit on the same P'; the
weighted attention must match the oracle's weighted attention within the
attention tolerance; and over many seeds the GPU's reweighted sum of exp terms
must average to the dense one.
"""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_45_b200 import binding as bsa
from block_sparse_attention_45_b200 import synth
from tests import checkers
from tests.gpu_util import sample_rows

pytestmark = pytest.mark.gpu

CASES = {
    "tiny": synth.WORKLOADS["tiny"],
    "small": synth.WORKLOADS["small"],
    "h3_b2": synth.custom("h3_b2", batch=2, heads=3, head_dim=64, q_block=128, k_block=64,
                          text_len=100, num_frames=3, latent_h=10, latent_w=16, top_p=0.8,
                          seed=31),                                      # gathered 64-key tiles
    "h5_d128": synth.custom("h5_d128", heads=5, head_dim=128, q_block=64, k_block=128,
                            text_len=40, num_frames=3, latent_h=10, latent_w=10, top_p=0.7,
                            seed=32),
}

_CACHE = {}


def _inputs(name):
    if name not in _CACHE:
        w = CASES[name]
        x = synth.generate(w)
        ora = oracle.default()
        L = w.layout()
        qc = ora.pool(L, x["q"], w.q_block)
        kc = ora.pool(L, x["k"], w.k_block)
        _CACHE[name] = (w, x, ora.scores(L, qc, kc))
    return _CACHE[name]


def _dev_bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)


def _compact(mask, weight):
    """Ascending lists of the mask's columns with their weights (oracle side)."""
    B, H, Cq, Ck = mask.shape
    idx = np.zeros((B, H, Cq, Ck), np.int32)
    wts = np.zeros((B, H, Cq, Ck), np.float32)
    cnt = mask.sum(-1).astype(np.int32)
    for r, (m, wr) in enumerate(zip(mask.reshape(-1, Ck), weight.reshape(-1, Ck))):
        js = np.nonzero(m)[0]
        idx.reshape(-1, Ck)[r, :len(js)] = js
        wts.reshape(-1, Ck)[r, :len(js)] = wr[js]
    return idx, wts, cnt


@pytest.mark.parametrize("seed", [0, 12345, 2**63 + 5])
@pytest.mark.parametrize("budget", [0.0, 2.0, 12.0, 1e9])
@pytest.mark.parametrize("name", sorted(CASES))
def test_sampler_bit_exact(name, budget, seed):
    w, _, probs = _inputs(name)
    ora = oracle.default()
    L = w.layout()
    for flags in (0, w.flags):
        m_o, w_o = ora.sample_select(L, probs, budget, seed, flags)
        g = bsa.build_mask_sampled(w, torch.from_numpy(probs).cuda(), budget, seed, flags)
        torch.cuda.synchronize()
        m_g = g["mask"].cpu().numpy()
        assert np.array_equal(m_g, m_o), (name, budget, seed, flags, np.argwhere(m_g != m_o)[:5])
        idx_o, wts_o, cnt_o = _compact(m_o, w_o)
        cnt_g = g["kv_count"].cpu().numpy()
        assert np.array_equal(cnt_g, cnt_o)
        idx_g = g["kv_index"].cpu().numpy()
        wts_g = g["kv_weight"].cpu().numpy()
        for r in range(cnt_o.size):
            n = cnt_o.reshape(-1)[r]
            assert np.array_equal(idx_g.reshape(-1, idx_g.shape[-1])[r, :n],
                                  idx_o.reshape(-1, idx_o.shape[-1])[r, :n])
            assert np.array_equal(wts_g.reshape(-1, wts_g.shape[-1])[r, :n],
                                  wts_o.reshape(-1, wts_o.shape[-1])[r, :n])


@pytest.mark.parametrize("budget", [3.0, 20.0])
@pytest.mark.parametrize("name", sorted(CASES))
def test_weighted_attention_parity(name, budget):
    w, x, probs = _inputs(name)
    ora = oracle.default()
    L = w.layout()
    m_o, w_o = ora.sample_select(L, probs, budget, 99, w.flags)
    idx, wts, cnt = _compact(m_o, w_o)
    q, k, v = _dev_bf16(x["q"]), _dev_bf16(x["k"]), _dev_bf16(x["v"])
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = bsa.attention_fwd_weighted(w, q, k, v, torch.from_numpy(idx).cuda(),
                                          torch.from_numpy(wts).cuda(), torch.from_numpy(cnt).cuda(),
                                          err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    o_ora, l_ora = ora.attention(L, x["q"], x["k"], x["v"], m_o, weight=w_o)
    B, H, Sp, D = w.batch, w.heads, w.seq_pad, w.head_dim
    o_ora = o_ora.reshape(B, H, Sp, D)
    l_ora = l_ora.reshape(B, H, Sp)
    o_g = out.float().cpu().numpy()
    l_g = lse.cpu().numpy()
    valid = np.arange(Sp) < w.seq_len
    d = np.abs(o_g[:, :, valid] - o_ora[:, :, valid])
    assert d.max() <= checkers.MAX_ABS and d.mean() <= checkers.MEAN_ABS, (d.max(), d.mean())
    fin = np.isfinite(l_ora[:, :, valid])
    np.testing.assert_array_equal(np.isfinite(l_g[:, :, valid]), fin)
    np.testing.assert_allclose(l_g[:, :, valid][fin], l_ora[:, :, valid][fin], rtol=1e-4,
                               atol=checkers.LSE_ABS)


@pytest.mark.parametrize("name", ["small", "h3_b2"])
def test_unit_weights_equal_the_unweighted_kernel(name):
    w, x, probs = _inputs(name)
    g = bsa.build_mask_sampled(w, torch.from_numpy(probs).cuda(), 6.0, 5, w.flags)
    q, k, v = _dev_bf16(x["q"]), _dev_bf16(x["k"]), _dev_bf16(x["v"])
    ones = torch.ones_like(g["kv_weight"])
    o1, l1 = bsa.attention_fwd_weighted(w, q, k, v, g["kv_index"], ones, g["kv_count"])
    o2, l2 = bsa.attention_fwd(w, q, k, v, g["kv_index"], g["kv_count"])
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)
    assert torch.equal(torch.nan_to_num(l1, neginf=-1e30), torch.nan_to_num(l2, neginf=-1e30))


def _block_constant(x, w):
    """Q and K constant inside every query / key block (V left as drawn): then a
    token's attention mass on key block j is exactly P'_ij, so the reweighted
    sum has relative variance sum_j P'_j (1 - pi_j) / (K) <= 1/K and no heavy
    tail -- a fair ground for a statistical check."""
    q = x["q"].copy()
    k = x["k"].copy()
    for arr, blk in ((q, w.q_block), (k, w.k_block)):
        for b0 in range(0, w.seq_pad, blk):
            arr[:, :, b0:b0 + blk] = arr[:, :, b0:b0 + 1]
    return q, k


def test_reweighted_sum_is_unbiased_on_the_gpu():
    """Over 400 seeds the mean of exp(lse_sampled - lse_dense) -- the reweighted
    sum of exp terms over the dense one -- is 1 within 5 standard errors on
    (almost) every valid query row, and 1 within 1 % on average: the GPU sampler
    feeding the GPU weighted kernel, end to end."""
    w = CASES["small"]
    x = synth.generate(w)
    qb, kb = _block_constant(x, w)
    ora = oracle.default()
    L = w.layout()
    probs = ora.scores(L, ora.pool(L, qb, w.q_block), ora.pool(L, kb, w.k_block))
    q, k, v = _dev_bf16(qb), _dev_bf16(kb), _dev_bf16(x["v"])
    P = torch.from_numpy(probs).cuda()
    _, l_dense = bsa.dense_fwd(w, q, k, v)
    valid = torch.arange(w.seq_pad, device="cuda") < w.seq_len
    n = 400
    acc = torch.zeros_like(l_dense, dtype=torch.float64)
    acc2 = torch.zeros_like(acc)
    for seed in range(n):
        g = bsa.build_mask_sampled(w, P, 16.0, 1000 + seed, 0, with_mask=False)
        _, l = bsa.attention_fwd_weighted(w, q, k, v, g["kv_index"], g["kv_weight"], g["kv_count"])
        r = torch.exp((l.double() - l_dense.double()).clamp(max=60))
        r = torch.where(torch.isfinite(l), r, torch.zeros_like(r))
        acc += r
        acc2 += r * r
    torch.cuda.synchronize()
    mean = acc / n
    se = torch.sqrt(torch.clamp(acc2 / n - mean * mean, min=0) / n)
    m = mean[..., valid]
    s = se[..., valid]
    z = (m - 1).abs() / torch.clamp(s, min=1e-6)
    # rows of one query block share their draws, so z is correlated across a block's tokens;
    # the bf16 kernel's lse error (~1e-3) is far inside the sampling noise (~1e-2)
    assert float((z > 5).double().mean()) < 0.005, float(z.max())
    assert abs(float(m.mean()) - 1) < 0.01, float(m.mean())
    # and the weights (all >= 1) are applied: on one draw the weighted sum is never below the
    # plain sum over the same blocks, and above it wherever a block with pi < 1 was drawn
    g = bsa.build_mask_sampled(w, P, 16.0, 7, 0, with_mask=False)
    _, l_w = bsa.attention_fwd_weighted(w, q, k, v, g["kv_index"], g["kv_weight"], g["kv_count"])
    _, l_plain = bsa.attention_fwd(w, q, k, v, g["kv_index"], g["kv_count"])
    fin = torch.isfinite(l_plain[..., valid])
    diff = (l_w - l_plain)[..., valid][fin]
    assert float(diff.min()) > -1e-3 and float(diff.mean()) > 0.01


def test_weighted_attention_full_size_sampled_rows():
    """Wan2.1-14B at full size (40 heads, 64-key blocks gathered into 128-key tiles):
    the GPU sampler's lists and weights feed the weighted kernel; the sampled query
    blocks (every frame-0 block of head 0, the ragged last block, 64 random ones
    spread over every head) match the oracle's weighted attention on the same lists."""
    w = synth.WORKLOADS["wan14b"]
    x = synth.generate(w)
    ora = oracle.default()
    L = w.layout()
    q, k, v = _dev_bf16(x["q"]), _dev_bf16(x["k"]), _dev_bf16(x["v"])
    _, _, probs = bsa.block_scores(w, q, k)
    g = bsa.build_mask_sampled(w, probs, 40.0, 2024, w.flags)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = bsa.attention_fwd_weighted(w, q, k, v, g["kv_index"], g["kv_weight"], g["kv_count"],
                                          err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    m_g = g["mask"].cpu().numpy()
    wt = np.zeros(m_g.shape, np.float32)
    idx, cnt, wts = g["kv_index"].cpu().numpy(), g["kv_count"].cpu().numpy(), g["kv_weight"].cpu().numpy()
    B, H, Cq, Ck = m_g.shape
    rows = sample_rows(w, seed=5)
    for r in rows:
        b, h, i = r // (H * Cq), (r // Cq) % H, r % Cq
        n = cnt[b, h, i]
        wt[b, h, i, idx[b, h, i, :n]] = wts[b, h, i, :n]
    o_ora, l_ora = ora.attention(L, x["q"], x["k"], x["v"], m_g, rows=rows, weight=wt)
    og = out.float().cpu().numpy().reshape(B * H, Cq, w.q_block, w.head_dim)
    lg = lse.cpu().numpy().reshape(B * H, Cq, w.q_block)
    for n_r, r in enumerate(rows):
        bh, i = r // Cq, r % Cq
        valid = np.arange(w.q_block) + i * w.q_block < w.seq_len
        d = np.abs(og[bh, i][valid] - o_ora[n_r][valid])
        assert d.max() <= checkers.MAX_ABS and d.mean() <= checkers.MEAN_ABS, (r, d.max(), d.mean())
        fin = np.isfinite(l_ora[n_r][valid])
        np.testing.assert_allclose(lg[bh, i][valid][fin], l_ora[n_r][valid][fin], rtol=1e-4,
                                   atol=checkers.LSE_ABS)
