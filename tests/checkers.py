"""Comparison rules between the CUDA path and the oracle.

Masks: a row whose oracle top-p decision has a margin above MARGIN must match
bit for bit; a row closer to the cut than that may differ by rounding, and
must then still be a valid top-p set (size within one of k*, mass >= p - MARGIN,
and without its smallest member, mass < p + MARGIN).  The margin of row i is
    min(p - c_{k*-1} (inf if k* = 1),  c_{k*} - p,  P'_(k*) - P'_(k*+1) (inf if k* = C_k))
with c_k the fp64 running sum of the row sorted by (P' desc, j asc).

Attention: given identical masks, the bf16 output must be within MAX_ABS of
the fp64-computed fp32 oracle at every element and MEAN_ABS on average; the
log-sum-exp within LSE_ABS.  Entropy within ENTROPY_REL relative.
"""
import itertools

import numpy as np

MARGIN = 1e-4            # end to end (GPU P' vs oracle P'): all three margin terms
MAX_ABS = 2e-2
MEAN_ABS = 2e-3
LSE_ABS = 1e-3
ENTROPY_REL = 1e-3


def row_margins(probs, top_p):
    """k* and the margin of every row of probs [B,H,Cq,Ck] (oracle fp32 values):
    min(p - c_{k*-1}, c_{k*} - p, P'_(k*) - P'_(k*+1))."""
    B, H, Cq, Ck = probs.shape
    tp = np.broadcast_to(np.asarray(top_p, np.float64), (H,))
    kstar = np.empty((B, H, Cq), np.int64)
    margin = np.empty((B, H, Cq), np.float64)
    order_all = np.argsort(-probs.astype(np.float64), axis=-1, kind="stable")
    for b in range(B):
        for h in range(H):
            p = np.float64(np.float32(tp[h]))
            srt = np.take_along_axis(probs[b, h].astype(np.float64), order_all[b, h], axis=-1)
            c = np.cumsum(srt, axis=-1)
            reach = c >= p
            k = np.where(reach.any(-1), reach.argmax(-1) + 1, Ck)
            kstar[b, h] = k
            idx = np.arange(Cq)
            ck = c[idx, k - 1]
            ckm1 = np.where(k > 1, c[idx, np.maximum(k - 2, 0)], -np.inf)
            gap = np.where(k < Ck, srt[idx, k - 1] - srt[idx, np.minimum(k, Ck - 1)], np.inf)
            m1 = np.where(k > 1, p - ckm1, np.inf)
            m2 = np.where(reach.any(-1), ck - p, np.inf)
            margin[b, h] = np.minimum(np.minimum(m1, m2), gap)
    return kstar, margin


def check_topp_masks(gpu_mask, ora_mask, probs, top_p, same_probs=False):
    """Compare top-p masks (no overrides).  Returns the exempt fraction.

    same_probs=True: the GPU read the oracle's own P'.  Both sides then sum
    exactly (the oracle's fp64 running sum of fp32 values spans fewer than 53
    bits down to any cut above 2^-29; the GPU sums integer significands per
    binade), so every row must match bit for bit.  Otherwise the end-to-end
    rule: bit-exact where the margin exceeds MARGIN (all three terms), a valid
    top-p set elsewhere."""
    if same_probs:
        gpu_b, ora_b = gpu_mask.astype(bool), ora_mask.astype(bool)
        bad = np.argwhere((gpu_b != ora_b).any(-1))
        assert bad.size == 0, "rows differ on identical P': %s (of %d)" % (bad[:5].tolist(), len(bad))
        return 0.0
    thr = MARGIN
    kstar, margin = row_margins(probs, top_p)
    gpu_mask = gpu_mask.astype(bool)
    ora_mask = ora_mask.astype(bool)
    strict = margin > thr
    diff = (gpu_mask != ora_mask).any(-1)
    bad = np.argwhere(diff & strict)
    assert bad.size == 0, "rows with margin > %g differ: %s (of %d)" % (thr, bad[:5].tolist(), len(bad))
    H = probs.shape[1]
    tp = np.broadcast_to(np.asarray(top_p, np.float64), (H,))
    for b, h, i in np.argwhere(diff & ~strict):
        p = np.float64(np.float32(tp[h]))
        row = probs[b, h, i].astype(np.float64)
        sel = np.nonzero(gpu_mask[b, h, i])[0]
        k = kstar[b, h, i]
        assert abs(len(sel) - k) <= 1, (b, h, i, len(sel), k)
        mass = row[sel].sum()
        assert mass >= p - MARGIN, (b, h, i, mass, p)
        assert mass - row[sel].min() < p + MARGIN, (b, h, i, mass, p)
    return float((~strict).mean())


def check_lists(kv_index, kv_count, mask):
    """kv_index/kv_count must be the ascending compaction of mask."""
    kv_index = np.asarray(kv_index)
    kv_count = np.asarray(kv_count)
    mask = np.asarray(mask).astype(bool)
    assert np.array_equal(kv_count, mask.sum(-1))
    Ck = mask.shape[-1]
    pos = np.arange(Ck)
    valid = pos < kv_count[..., None]
    ref = np.sort(np.where(mask, pos, Ck), axis=-1)
    assert np.array_equal(np.where(valid, kv_index, -1), np.where(valid, ref, -1))


def bf16_output_bound(out_ora, v_max):
    """Largest max-abs error bf16 arithmetic can produce at this value range:
    output rounding (2^-9 |o|) plus the rounding of P to bf16 before the PV
    product, which perturbs each normalised weight by at most 2^-8 relative
    (<= 2^-8 max|V|).  The spec's MAX_ABS applies when this is below it."""
    return max(MAX_ABS, 2.0 ** -9 * float(np.abs(out_ora).max()) + 2.0 ** -8 * float(v_max))


def check_attention(out_gpu, out_ora, lse_gpu=None, lse_ora=None, what="", max_abs=MAX_ABS):
    out_gpu = np.asarray(out_gpu, np.float64)
    out_ora = np.asarray(out_ora, np.float64)
    assert np.isfinite(out_gpu).all(), what + ": non-finite output"
    err = np.abs(out_gpu - out_ora)
    assert err.max() <= max_abs, "%s: max abs err %.3g > %g" % (what, err.max(), max_abs)
    assert err.mean() <= MEAN_ABS, "%s: mean abs err %.3g > %g" % (what, err.mean(), MEAN_ABS)
    if lse_gpu is not None:
        lg = np.asarray(lse_gpu, np.float64)
        lo = np.asarray(lse_ora, np.float64)
        fin = np.isfinite(lo)
        assert np.array_equal(fin, np.isfinite(lg)), what + ": lse finiteness differs"
        if fin.any():
            e = np.abs(lg[fin] - lo[fin]).max()
            assert e <= LSE_ABS, "%s: lse err %.3g" % (what, e)
    return float(err.max()), float(err.mean())


def kmeans_end_states(x, n_sub, iters, rel=1e-4, cap=4096):
    """(centroids, sizes) of every end state of the k-means rounds on the block's
    tokens x [n, D] (fp64) when a token whose squared distance to a centroid is
    within rel * (|x|^2 + max |c|^2) of its nearest may be assigned to it.  Seeds,
    the move step and empty clusters follow the oracle's k-means."""
    n, D = x.shape
    xx = (x * x).sum(1)
    c0 = np.stack([x[(k * n) // n_sub] if n > 0 else np.zeros(D) for k in range(n_sub)])
    states = [(c0, np.zeros(n_sub, np.int64))]
    for _ in range(iters):
        nxt = {}
        for c, _sizes in states:
            d = ((x[:, None, :] - c[None, :, :]) ** 2).sum(-1)
            dmin = d.min(1)
            tol = rel * (xx + (c * c).sum(1).max())
            cands = [np.nonzero(d[t] <= dmin[t] + tol[t])[0] for t in range(n)]
            amb = [t for t in range(n) if len(cands[t]) > 1]
            n_combos = int(np.prod([len(cands[t]) for t in amb])) if amb else 1
            assert n_combos <= cap, "too many near-equidistant tokens to replay (%d)" % n_combos
            base = d.argmin(1)
            for combo in itertools.product(*[cands[t] for t in amb]):
                a = base.copy()
                a[amb] = combo
                sizes = np.bincount(a, minlength=n_sub)
                cn = c.copy()
                for k in range(n_sub):
                    if sizes[k] > 0:
                        cn[k] = x[a == k].mean(0)
                nxt[a.tobytes() + cn[sizes == 0].tobytes()] = (cn, sizes)
        states = list(nxt.values())
        assert len(states) <= cap, "too many branches to replay (%d)" % len(states)
    return states
