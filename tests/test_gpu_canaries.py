"""Guard canaries around every output and workspace of the entry points that the
pipeline and parity tests do not already guard (needs a B200).

Each buffer sits between 4 KB of a fixed byte pattern (tests.guard) that must be
intact after the call; the guarded call must also give the same results as the
same call on plain buffers, so every output byte it owns was written.  (The
allocation-free mask entry point has its canaries in its own test file.)  Shapes are
ragged (the last key and query blocks are partial) and cover both block sizes
and head dimensions: "Attention matrix view: make only frame-0 query rows
dense" s4 — block kernels write whole blocks, so a ragged last block is where an
overrun would land.
"""
import numpy as np
import pytest
import torch

from block_sparse_attention_45_b200 import binding as bsa
from block_sparse_attention_45_b200 import synth
from tests.gpu_util import to_dev
from tests.guard import Guard

pytestmark = pytest.mark.gpu

CASES = {
    "h3_b2": synth.custom("h3_b2", batch=2, heads=3, head_dim=64, q_block=128, k_block=64,
                          text_len=100, num_frames=3, latent_h=10, latent_w=16, top_p=0.8,
                          seed=31),
    "h5_d128": synth.custom("h5_d128", heads=5, head_dim=128, q_block=64, k_block=128,
                            text_len=40, num_frames=3, latent_h=10, latent_w=10, top_p=0.7,
                            seed=32),
}

_CACHE = {}


def _data(name):
    if name not in _CACHE:
        w = CASES[name]
        x = synth.generate(w)
        _CACHE[name] = (w, x, {k: to_dev(v) for k, v in x.items()})
    return _CACHE[name]


def _dims(w):
    return w.batch, w.heads, w.seq_pad // w.q_block, w.seq_pad // w.k_block


def _lists_equal(idx_a, cnt_a, idx_b, cnt_b):
    assert torch.equal(cnt_a, cnt_b)
    ck = idx_a.shape[-1]
    valid = torch.arange(ck, device=idx_a.device) < cnt_a[..., None]
    assert torch.equal(torch.where(valid, idx_a, -1), torch.where(valid, idx_b, -1))


@pytest.mark.parametrize("name", sorted(CASES))
def test_value_norms_and_pooled_selections(name):
    w, x, xd = _data(name)
    B, H, Cq, Ck = _dims(w)
    _, _, probs = bsa.block_scores(w, xd["q"], xd["k"])
    tp = [w.top_p] * H
    gd = Guard()
    vn = bsa.value_norms(w, xd["v"], gd.alloc((B, H, Ck), torch.float32, "vnorm"))
    gd.check()
    assert torch.equal(vn, bsa.value_norms(w, xd["v"]))

    def guarded(tag, ws_bytes):
        return dict(mask=gd.alloc((B, H, Cq, Ck), torch.uint8, tag + " mask"),
                    kv_index=gd.alloc((B, H, Cq, Ck), torch.int32, tag + " kv_index"),
                    kv_count=gd.alloc((B, H, Cq), torch.int32, tag + " kv_count"),
                    entropy=gd.alloc((B, H), torch.float32, tag + " entropy"),
                    entropy_norm=gd.alloc((B, H), torch.float32, tag + " entropy_norm"),
                    workspace=gd.bytes(ws_bytes, tag + " workspace"))

    g = bsa.build_mask_eg(w, probs, vn, tp, 0.8, w.flags, low_heads=gd.alloc(
        (B, H), torch.uint8, "low_heads"), **guarded("eg", bsa.eg_workspace_bytes(w)))
    gd.check()
    r = bsa.build_mask_eg(w, probs, vn, tp, 0.8, w.flags)
    for key in ("mask", "entropy", "entropy_norm", "low_heads"):
        assert torch.equal(g[key], r[key]), key
    _lists_equal(g["kv_index"], g["kv_count"], r["kv_index"], r["kv_count"])

    for dom in (bsa.DOMAIN_ROW, bsa.DOMAIN_HEAD, bsa.DOMAIN_GROUPED, bsa.DOMAIN_ALL, bsa.DOMAIN_EG):
        tag = "domain %d" % dom
        g = bsa.build_mask_domain(w, dom, probs, vn, tp, 0.8, w.flags, pool_of=gd.alloc(
            (B, H), torch.int8, tag + " pool_of"), **guarded(tag, bsa.domain_workspace_bytes(w, dom)))
        gd.check()
        r = bsa.build_mask_domain(w, dom, probs, vn, tp, 0.8, w.flags)
        for key in ("mask", "entropy", "entropy_norm", "pool_of"):
            assert torch.equal(g[key], r[key]), (dom, key)
        _lists_equal(g["kv_index"], g["kv_count"], r["kv_index"], r["kv_count"])


@pytest.mark.parametrize("name", sorted(CASES))
def test_sampler_and_weighted_attention(name):
    w, x, xd = _data(name)
    B, H, Cq, Ck = _dims(w)
    Sp, D = w.seq_pad, w.head_dim
    _, _, probs = bsa.block_scores(w, xd["q"], xd["k"])
    gd = Guard()
    g = bsa.build_mask_sampled(w, probs, 3.0, 77, w.flags,
                               mask=gd.alloc((B, H, Cq, Ck), torch.uint8, "mask"),
                               kv_index=gd.alloc((B, H, Cq, Ck), torch.int32, "kv_index"),
                               kv_weight=gd.alloc((B, H, Cq, Ck), torch.float32, "kv_weight"),
                               kv_count=gd.alloc((B, H, Cq), torch.int32, "kv_count"))
    gd.check()
    r = bsa.build_mask_sampled(w, probs, 3.0, 77, w.flags)
    assert torch.equal(g["mask"], r["mask"])
    _lists_equal(g["kv_index"], g["kv_count"], r["kv_index"], r["kv_count"])
    valid = torch.arange(Ck, device="cuda") < g["kv_count"][..., None]
    assert torch.equal(torch.where(valid, g["kv_weight"], 0.0), torch.where(valid, r["kv_weight"], 0.0))
    err = gd.alloc((1,), torch.int32, "err_flag")
    err.zero_()
    out, lse = bsa.attention_fwd_weighted(
        w, xd["q"], xd["k"], xd["v"], r["kv_index"], r["kv_weight"], r["kv_count"],
        out=gd.alloc((B, H, Sp, D), torch.bfloat16, "out"),
        lse=gd.alloc((B, H, Sp), torch.float32, "lse"), err_flag=err,
        workspace=gd.bytes(bsa.attention_workspace_bytes(w), "workspace"))
    gd.check()
    assert int(err.item()) == 0
    o2, l2 = bsa.attention_fwd_weighted(w, xd["q"], xd["k"], xd["v"], r["kv_index"],
                                        r["kv_weight"], r["kv_count"])
    torch.cuda.synchronize()
    assert torch.equal(out, o2)
    assert torch.equal(torch.nan_to_num(lse, nan=7.0), torch.nan_to_num(l2, nan=7.0))


@pytest.mark.parametrize("name", sorted(CASES))
def test_clustered_scores(name):
    w, x, xd = _data(name)
    B, H, Cq, Ck = _dims(w)
    D = w.head_dim
    n_sub = 4
    gd = Guard()
    c, s, kc, p = bsa.block_scores_clustered(
        w, xd["q"], xd["k"], n_sub, 2,
        sub_centroids=gd.alloc((B, H, Cq, n_sub, D), torch.float32, "sub_centroids"),
        sub_sizes=gd.alloc((B, H, Cq, n_sub), torch.int32, "sub_sizes"),
        k_centroids=gd.alloc((B, H, Ck, D), torch.float32, "k_centroids"),
        probs=gd.alloc((B, H, Cq, Ck), torch.float32, "probs"),
        workspace=gd.bytes(bsa.clustered_workspace_bytes(w, n_sub), "workspace"))
    gd.check()
    c2, s2, kc2, p2 = bsa.block_scores_clustered(w, xd["q"], xd["k"], n_sub, 2)
    torch.cuda.synchronize()
    for a, b in ((c, c2), (s, s2), (kc, kc2), (p, p2)):
        assert torch.equal(a, b)


def test_frame_scores():
    w = synth.custom("f3_d64_ragged", heads=3, head_dim=64, num_frames=3, latent_h=10, latent_w=16,
                     q_block=64, k_block=128, seed=42, kind="clustered", sigma_mean=2.0)
    x = synth.generate(w, ("q", "k"))
    q, k = to_dev(x["q"]), to_dev(x["k"])
    gd = Guard()
    alpha = bsa.frame_scores(w, q, k, alpha=gd.alloc((w.batch, w.heads, 3), torch.float32, "alpha"),
                             workspace=gd.bytes(bsa.frame_scores_workspace_bytes(w), "workspace"))
    gd.check()
    assert torch.equal(alpha, bsa.frame_scores(w, q, k))


def test_host_pipeline_workspace():
    w, x, xd = _data("h3_b2")
    B, H, Cq, Ck = _dims(w)
    host = {n: torch.from_numpy(x[n].view(np.int16)).view(torch.bfloat16).pin_memory()
            for n in ("q", "k", "v")}
    gd = Guard()
    nb = bsa.pipeline_workspace_bytes(w, 2)
    res = bsa.sparse_attention_host(w, host["q"], host["k"], host["v"], [w.top_p] * H, w.flags,
                                    heads_per_group=2, workspace=gd.bytes(nb, "workspace"))
    torch.cuda.current_stream().synchronize()
    gd.check()
    ref = bsa.sparse_attention(w, xd["q"], xd["k"], xd["v"], [w.top_p] * H, w.flags)
    torch.cuda.synchronize()
    assert torch.equal(res["out"], ref["out"].cpu())

