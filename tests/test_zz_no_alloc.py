"""bsa_build_mask_noalloc against bsa_build_mask (needs a B200).

bsa_build_mask_noalloc exists for callers that cannot allocate device memory
(a framework allocator or memory-planning pass, a process whose device memory
is reserved up front, a plugin whose host owns every allocation) and so have no
workspace to pass: it keeps the per-row entropies in an array inside the
library.  These tests call it through the C ABI twice in a row, on two
different geometries, and require the same masks, lists and entropies as the
ordinary entry point given a workspace; they check that a problem larger than
the array is refused when entropies are asked for, and that without entropies
(no workspace needed) such a problem runs and matches the ordinary entry point.

This file is collected last on purpose; it works alone in a fresh process too.
"""
import ctypes

import numpy as np
import pytest
import torch

from block_sparse_attention_45_b200 import binding as bsa
from block_sparse_attention_45_b200 import synth
from tests import checkers

pytestmark = pytest.mark.gpu


def _probs(name):
    w = synth.WORKLOADS[name]
    x = synth.generate(w, ("q", "k"))
    to = lambda a: torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)  # noqa: E731
    _, _, probs = bsa.block_scores(w, to(x["q"]), to(x["k"]))
    return w, probs


def _noalloc(w, probs, top_p, flags, with_entropy=True):
    L = bsa.make_layout(w)
    d = bsa.dims(L)
    B, H, cq, ck = d["B"], d["H"], d["Cq"], d["Ck"]
    dev = probs.device
    mask = torch.full((B, H, cq, ck), 7, dtype=torch.uint8, device=dev)
    idx = torch.full((B, H, cq, ck), -5, dtype=torch.int32, device=dev)
    cnt = torch.full((B, H, cq), -5, dtype=torch.int32, device=dev)
    ent = entn = None
    if with_entropy:
        ent = torch.full((B, H), float("nan"), dtype=torch.float32, device=dev)
        entn = torch.full((B, H), float("nan"), dtype=torch.float32, device=dev)
    ptr = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())  # noqa: E731
    tp = (ctypes.c_float * H)(*top_p)
    rc = bsa.load().bsa_build_mask_noalloc(
        ctypes.byref(L), ptr(probs), ctypes.cast(tp, ctypes.c_void_p), flags, 1e-8, ptr(mask),
        ptr(idx), ptr(cnt), ptr(ent), ptr(entn),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == bsa.BSA_OK, bsa.status_string(rc)
    return dict(mask=mask, kv_index=idx, kv_count=cnt, entropy=ent, entropy_norm=entn)


def _same(a, b):
    torch.cuda.synchronize()
    assert torch.equal(a["mask"], b["mask"])
    assert torch.equal(a["kv_count"], b["kv_count"])
    m = b["mask"].cpu().numpy()
    checkers.check_lists(a["kv_index"].cpu().numpy(), a["kv_count"].cpu().numpy(), m)
    for k in ("entropy", "entropy_norm"):
        if b[k] is not None:
            np.testing.assert_allclose(a[k].cpu().numpy(), b[k].cpu().numpy(),
                                       rtol=checkers.ENTROPY_REL)


def test_noalloc_matches_workspace_entry_point_twice():
    # two calls in a row with different geometries: the second must not see the first's scratch
    for name in ("small", "tiny"):
        w, probs = _probs(name)
        tp = [float(w.top_p)] * w.heads
        ref = bsa.build_mask(w, probs, tp, w.flags)
        got = _noalloc(w, probs, tp, w.flags)
        _same(got, ref)


def test_noalloc_rejects_problems_larger_than_its_array():
    w = synth.WORKLOADS["hunyuan"]
    d = w.layout()
    d["batch"] = 12            # 12 * 24 * 931 rows > 262144
    L = bsa.make_layout(d)
    # Only `entropy` is non-null (a dummy that is never dereferenced): it is what
    # makes the call need the array.  Should the size check ever stop refusing,
    # the null probs / lists make bsa_build_mask reject the call before any launch.
    dummy = ctypes.c_void_p(0x10000)
    tp = (ctypes.c_float * w.heads)(*([0.9] * w.heads))
    rc = bsa.load().bsa_build_mask_noalloc(ctypes.byref(L), None, ctypes.cast(tp, ctypes.c_void_p),
                                           3, 1e-8, None, None, None, dummy, None, None)
    assert rc == bsa.BSA_ERR_UNSUPPORTED


def test_noalloc_without_entropy_is_not_capped():
    """Masks and lists only: no workspace is needed, so a problem with more rows
    than the array runs, twice in a row, and matches bsa_build_mask."""
    layout = dict(batch=64, heads=66, seq_len=4096, seq_pad=4096, head_dim=64, q_block=64,
                  k_block=128, text_len=0, tokens_per_frame=0, num_frames=0)
    d = bsa.dims(bsa.make_layout(layout))
    assert d["B"] * d["H"] * d["Cq"] > 262144
    g = torch.Generator(device="cuda").manual_seed(5)
    x = torch.rand((d["B"], d["H"], d["Cq"], d["Ck"]), generator=g, device="cuda") ** 4
    probs = (x / x.sum(-1, keepdim=True)).contiguous()
    tp = [0.5 + 0.4 * (h % 5) / 4 for h in range(d["H"])]
    ref = bsa.build_mask(layout, probs, tp, 0, with_entropy=False)
    for _ in range(2):
        got = _noalloc(layout, probs, tp, 0, with_entropy=False)
        _same(got, ref)


def test_noalloc_writes_only_inside_its_buffers():
    """Every output sits between guard canaries that must stay intact."""
    from tests.guard import Guard
    w, probs = _probs("small")
    B, H = w.batch, w.heads
    cq, ck = w.seq_pad // w.q_block, w.seq_pad // w.k_block
    gd = Guard()
    outs = dict(mask=gd.alloc((B, H, cq, ck), torch.uint8, "mask"),
                kv_index=gd.alloc((B, H, cq, ck), torch.int32, "kv_index"),
                kv_count=gd.alloc((B, H, cq), torch.int32, "kv_count"),
                entropy=gd.alloc((B, H), torch.float32, "entropy"),
                entropy_norm=gd.alloc((B, H), torch.float32, "entropy_norm"))
    ptr = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    tp = [float(w.top_p)] * H
    tpc = (ctypes.c_float * H)(*tp)
    rc = bsa.load().bsa_build_mask_noalloc(
        ctypes.byref(bsa.make_layout(w)), ptr(probs), ctypes.cast(tpc, ctypes.c_void_p), w.flags,
        1e-8, ptr(outs["mask"]), ptr(outs["kv_index"]), ptr(outs["kv_count"]), ptr(outs["entropy"]),
        ptr(outs["entropy_norm"]), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == bsa.BSA_OK, bsa.status_string(rc)
    gd.check()
    _same(outs, bsa.build_mask(w, probs, tp, w.flags))
