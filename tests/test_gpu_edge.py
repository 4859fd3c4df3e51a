"""Edge cases of the CUDA path against the oracle (needs a B200).

Ragged sequence ends, every (head_dim, q_block, k_block) combination, text and
frame 0 that start or end inside a block, hand-built lists (one block, every
block, none, odd counts in gather mode, invalid entries and counts) and
garbage in the padded rows.
"""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_45_b200 import binding as bsa
from block_sparse_attention_45_b200 import synth
from tests import checkers
from tests.gpu_util import to_dev, to_host_f32
from tests.guard import Guard

pytestmark = pytest.mark.gpu

EDGE = {
    # D, bq, bk, text_len, frames, latent (h, w), pad_to  -> seq_len, seq_pad
    "d128_q64_k128": synth.custom("d128_q64_k128", heads=3, head_dim=128, q_block=64, k_block=128,
                                  text_len=40, num_frames=3, latent_h=10, latent_w=10, top_p=0.8,
                                  seed=11),                                  # 340 -> 384
    "d128_q128_k64": synth.custom("d128_q128_k64", heads=2, head_dim=128, q_block=128, k_block=64,
                                  text_len=90, num_frames=4, latent_h=10, latent_w=16, top_p=0.75,
                                  seed=12),                                  # 730 -> 768
    "d64_q128_k128": synth.custom("d64_q128_k128", heads=2, head_dim=64, q_block=128, k_block=128,
                                  text_len=20, num_frames=3, latent_h=10, latent_w=16, top_p=0.85,
                                  seed=13),                                  # 500 -> 512
    "d64_q64_k64": synth.custom("d64_q64_k64", heads=2, head_dim=64, q_block=64, k_block=64,
                                text_len=10, num_frames=2, latent_h=6, latent_w=10, top_p=0.6,
                                pad_to=64, seed=14),                         # 130 -> 192
    "d128_q64_k64": synth.custom("d128_q64_k64", heads=2, head_dim=128, q_block=64, k_block=64,
                                 text_len=33, num_frames=3, latent_h=7, latent_w=9, top_p=0.8,
                                 pad_to=64, seed=16),                        # 222 -> 256
    "d64_q64_k128": synth.custom("d64_q64_k128", heads=2, head_dim=64, q_block=64, k_block=128,
                                 text_len=70, num_frames=2, latent_h=10, latent_w=20, top_p=0.7,
                                 seed=17),                                   # 470 -> 512
    "d64_q128_k64": synth.custom("d64_q128_k64", batch=2, heads=2, head_dim=64, q_block=128,
                                 k_block=64, text_len=0, num_frames=5, latent_h=9, latent_w=22,
                                 top_p=0.7, seed=15, kind="clustered"),      # 990 -> 1024
}


def _data(w):
    x = synth.generate(w)
    return x, {k: to_dev(v) for k, v in x.items()}


def _attn_vs_oracle(w, x, xd, mask, idx, cnt, what, gd=None):
    L = w.layout()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    outs = {}
    if gd is not None:
        B, H, Sp, D = w.batch, w.heads, w.seq_pad, w.head_dim
        outs = dict(out=gd.alloc((B, H, Sp, D), torch.bfloat16, what + " out"),
                    lse=gd.alloc((B, H, Sp), torch.float32, what + " lse"),
                    workspace=gd.bytes(bsa.attention_workspace_bytes(w), what + " workspace"))
    out, lse = bsa.attention_fwd(w, xd["q"], xd["k"], xd["v"], torch.from_numpy(idx).cuda(),
                                 torch.from_numpy(cnt).cuda(), err_flag=err, **outs)
    torch.cuda.synchronize()
    if gd is not None:
        gd.check()
    o_ora, l_ora = oracle.attention(L, x["q"], x["k"], x["v"], mask)
    cq = w.seq_pad // w.q_block
    og = to_host_f32(out).reshape(o_ora.shape)
    lg = lse.cpu().numpy().reshape(l_ora.shape)
    vmax = np.abs(synth.bf16_bits_to_f32(x["v"])).max()
    checkers.check_attention(og, o_ora, lg, l_ora, what=what,
                             max_abs=checkers.bf16_output_bound(o_ora, vmax))
    return out, lse, int(err.item())


def _mask_outputs(gd, w, tag):
    B, H = w.batch, w.heads
    cq, ck = w.seq_pad // w.q_block, w.seq_pad // w.k_block
    return dict(mask=gd.alloc((B, H, cq, ck), torch.uint8, tag + " mask"),
                kv_index=gd.alloc((B, H, cq, ck), torch.int32, tag + " kv_index"),
                kv_count=gd.alloc((B, H, cq), torch.int32, tag + " kv_count"),
                entropy=gd.alloc((B, H), torch.float32, tag + " entropy"),
                entropy_norm=gd.alloc((B, H), torch.float32, tag + " entropy_norm"),
                workspace=gd.bytes(bsa.workspace_bytes(w), tag + " workspace"))


@pytest.mark.parametrize("name", sorted(EDGE))
def test_pipeline_edge_shapes(name):
    """Every stage on a ragged shape, each output and workspace between guard canaries."""
    w = EDGE[name]
    x, xd = _data(w)
    L = w.layout()
    tp = [w.top_p] * w.heads
    B, H, Sp, D = w.batch, w.heads, w.seq_pad, w.head_dim
    cq, ck = Sp // w.q_block, Sp // w.k_block
    gd = Guard()
    sel = oracle.select(L, x["q"], x["k"], tp, w.flags)
    qc, kc, probs = bsa.block_scores(w, xd["q"], xd["k"],
                                     gd.alloc((B, H, cq, D), torch.float32, "q_centroids"),
                                     gd.alloc((B, H, ck, D), torch.float32, "k_centroids"),
                                     gd.alloc((B, H, cq, ck), torch.float32, "probs"))
    gd.check()
    np.testing.assert_allclose(to_host_f32(qc), sel["q_centroids"], rtol=1e-5, atol=2e-6)
    np.testing.assert_allclose(to_host_f32(kc), sel["k_centroids"], rtol=1e-5, atol=2e-6)
    assert np.abs(to_host_f32(probs) - sel["probs"]).max() <= 1e-4
    g0 = bsa.build_mask(w, torch.from_numpy(sel["probs"]).cuda(), tp, 0, **_mask_outputs(gd, w, "top-p"))
    gd.check()
    checkers.check_topp_masks(g0["mask"].cpu().numpy(), sel["topp_mask"], sel["probs"], tp,
                              same_probs=True)
    g = bsa.build_mask(w, torch.from_numpy(sel["probs"]).cuda(), tp, w.flags,
                       **_mask_outputs(gd, w, "overrides"))
    gd.check()
    m = g["mask"].cpu().numpy()
    assert np.array_equal(m, oracle.overrides(L, w.flags, g0["mask"].cpu().numpy()))
    checkers.check_lists(g["kv_index"].cpu().numpy(), g["kv_count"].cpu().numpy(), m)
    np.testing.assert_allclose(g["entropy"].cpu().numpy(), sel["entropy"], rtol=checkers.ENTROPY_REL)
    _attn_vs_oracle(w, x, xd, sel["mask"], sel["kv_index"], sel["kv_count"], name, gd)
    out, lse = bsa.dense_fwd(w, xd["q"], xd["k"], xd["v"],
                             out=gd.alloc((B, H, Sp, D), torch.bfloat16, "dense out"),
                             lse=gd.alloc((B, H, Sp), torch.float32, "dense lse"),
                             workspace=gd.bytes(bsa.attention_workspace_bytes(w), "dense workspace"))
    gd.check()
    o_ora, l_ora = oracle.attention(L, x["q"], x["k"], x["v"], None)
    vmax = np.abs(synth.bf16_bits_to_f32(x["v"])).max()
    checkers.check_attention(to_host_f32(out).reshape(o_ora.shape), o_ora,
                             lse.cpu().numpy().reshape(l_ora.shape), l_ora, what=name + " dense",
                             max_abs=checkers.bf16_output_bound(o_ora, vmax))


def _lists_from_mask(mask):
    Ck = mask.shape[-1]
    pos = np.arange(Ck)
    idx = np.sort(np.where(mask.astype(bool), pos, Ck), axis=-1).astype(np.int32)
    cnt = mask.astype(bool).sum(-1).astype(np.int32)
    idx[idx == Ck] = -1
    return idx, cnt


@pytest.mark.parametrize("name", ["d128_q128_k64", "d64_q64_k64", "d128_q64_k128"])
def test_hand_built_lists(name):
    w = EDGE[name]
    x, xd = _data(w)
    cq, ck = w.seq_pad // w.q_block, w.seq_pad // w.k_block
    rng = np.random.default_rng(7)
    shape = (w.batch, w.heads, cq, ck)
    # one block per row, including the ragged last key block
    m = np.zeros(shape, np.uint8)
    m[..., :] = 0
    js = rng.integers(ck, size=shape[:-1])
    js.reshape(-1)[0] = ck - 1
    np.put_along_axis(m, js[..., None], 1, axis=-1)
    _attn_vs_oracle(w, x, xd, m, *_lists_from_mask(m), what=name + " one block")
    # every block (equals dense)
    m = np.ones(shape, np.uint8)
    out, _, _ = _attn_vs_oracle(w, x, xd, m, *_lists_from_mask(m), what=name + " all blocks")
    dn, _ = bsa.dense_fwd(w, xd["q"], xd["k"], xd["v"])
    assert torch.equal(out, dn)
    # random counts: odd and even, 1..C_k
    m = (rng.random(shape) < 0.4).astype(np.uint8)
    m[..., 0, :] = 0
    m[..., 0, ck // 2] = 1
    _attn_vs_oracle(w, x, xd, m, *_lists_from_mask(m), what=name + " random")


def test_empty_rows_and_bad_entries():
    w = EDGE["d128_q128_k64"]
    x, xd = _data(w)
    cq, ck = w.seq_pad // w.q_block, w.seq_pad // w.k_block
    shape = (w.batch, w.heads, cq, ck)
    m = np.zeros(shape, np.uint8)
    m[..., 1:, :3] = 1          # query block 0 of every head selects nothing
    idx, cnt = _lists_from_mask(m)
    out, lse, e = _attn_vs_oracle(w, x, xd, m, idx, cnt, what="empty rows")
    assert e == 0
    assert (out[:, :, :w.q_block] == 0).all()
    assert torch.isneginf(lse[:, :, :w.q_block]).all()
    # invalid entries are skipped and flagged; counts beyond C_k are clamped and flagged
    idx2 = idx.copy()
    cnt2 = cnt.copy()
    idx2[0, 0, 1, 3] = ck + 5      # list of (0,0,1) = [0,1,2, bad]
    cnt2[0, 0, 1] = 4
    idx2[0, 1, 2, :4] = [0, -3, 1, 2]
    cnt2[0, 1, 2] = 4
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out2, _ = bsa.attention_fwd(w, xd["q"], xd["k"], xd["v"], torch.from_numpy(idx2).cuda(),
                                torch.from_numpy(cnt2).cuda(), err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) & bsa.DEVERR_BAD_INDEX
    assert torch.equal(out2[0, 0, w.q_block:2 * w.q_block], out[0, 0, w.q_block:2 * w.q_block])
    # a bad entry inside a gathered pair changes the pairing, so compare within tolerance
    a = out2[0, 1, 2 * w.q_block:3 * w.q_block].float()
    b = out[0, 1, 2 * w.q_block:3 * w.q_block].float()
    assert (a - b).abs().max().item() <= 2 * checkers.MAX_ABS
    cnt3 = np.full_like(cnt, ck + 7)
    err.zero_()
    out3, _ = bsa.attention_fwd(w, xd["q"], xd["k"], xd["v"],
                                torch.from_numpy(np.broadcast_to(np.arange(ck, dtype=np.int32),
                                                                 shape).copy()).cuda(),
                                torch.from_numpy(cnt3).cuda(), err_flag=err)
    dn, _ = bsa.dense_fwd(w, xd["q"], xd["k"], xd["v"])
    torch.cuda.synchronize()
    assert int(err.item()) & bsa.DEVERR_BAD_COUNT
    assert torch.equal(out3, dn)


def test_padding_rows_are_ignored_and_zeroed():
    w = EDGE["d64_q128_k128"]
    x, xd = _data(w)
    S = w.seq_len
    ref, ref_lse = bsa.dense_fwd(w, xd["q"], xd["k"], xd["v"])
    dirty = {k: v.clone() for k, v in xd.items()}
    for t in dirty.values():
        t[:, :, S:] = float("nan")
    out = torch.full_like(ref, float("nan"))
    lse = torch.full_like(ref_lse, 123.0)
    bsa.dense_fwd(w, dirty["q"], dirty["k"], dirty["v"], out=out, lse=lse)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
    assert (out[:, :, S:] == 0).all()
    assert torch.isneginf(lse[:, :, S:]).all()
    assert torch.equal(lse[:, :, :S], ref_lse[:, :, :S])


def _crafted_probs(rng, rows, ck):
    """P' rows that exercise every branch of the GPU cut search."""
    out = []
    for r in range(rows):
        kind = r % 8
        if kind == 0:                                    # generic
            x = rng.dirichlet(np.full(ck, 0.3))
        elif kind == 1:                                  # flat: one binade holds every entry
            x = np.full(ck, 1.0 / ck)
        elif kind == 2:                                  # flat with noise inside one binade
            x = (1.0 + 0.5 * rng.random(ck)) / ck
        elif kind == 3:                                  # many exact ties at the cut
            x = np.full(ck, 0.25 / ck)
            x[rng.choice(ck, 5, replace=False)] = 0.15
        elif kind == 4:                                  # very peaked with tiny tail values
            x = rng.random(ck) ** 12
            x[rng.integers(ck)] = 50.0
        elif kind == 5:                                  # two-level
            x = np.where(rng.random(ck) < 0.1, 1.0, 1e-3)
        elif kind == 6:                                  # some exact zeros
            x = rng.dirichlet(np.full(ck, 0.5))
            x[rng.random(ck) < 0.3] = 0.0
        else:                                            # a few equal maxima
            x = rng.random(ck) * 0.1
            x[:3] = 1.0
        x = np.asarray(x, np.float64)
        out.append((x / x.sum()).astype(np.float32))
    return np.stack(out)


@pytest.mark.parametrize("ck_blocks", [5, 64, 300, 931, 1500, 2048])
def test_topp_crafted_rows_exact(ck_blocks):
    """On identical fp32 P' the GPU top-p must equal the oracle's row for row:
    both sum in fp64 in the same order-independent way at the cut."""
    rng = np.random.default_rng(ck_blocks)
    L = dict(batch=1, heads=4, seq_len=ck_blocks * 128, seq_pad=ck_blocks * 128, head_dim=128,
             q_block=128, k_block=128, text_len=0, tokens_per_frame=0, num_frames=0)
    cq = L["seq_pad"] // L["q_block"]
    probs = _crafted_probs(rng, 4 * cq, ck_blocks).reshape(1, 4, cq, ck_blocks)
    for tp in ([0.5, 0.9, 0.99, 0.999999], [1e-9, 0.3, 1.0, 2.0], [-1.0, 0.7, 0.75, 0.8]):
        m_ora, _ = oracle.topp(L, probs, tp)
        g = bsa.build_mask(L, torch.from_numpy(probs).cuda(), tp, 0)
        torch.cuda.synchronize()
        got = g["mask"].cpu().numpy()
        bad = np.argwhere((got != m_ora).any(-1))
        assert bad.size == 0, (tp, bad[:5].tolist())
        checkers.check_lists(g["kv_index"].cpu().numpy(), g["kv_count"].cpu().numpy(), got)
