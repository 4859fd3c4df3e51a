"""bsa_sparse_attention_host against the three device entry points (needs a B200).

The pipelined host entry point must give exactly what bsa_block_scores ->
bsa_build_mask -> bsa_attention_fwd give on the same data: the same kernels
run per head group, and every per-head result (P', lists, entropy, attention)
depends on that head alone.  Cases cover a ragged last group, a batch of two,
one shared stream and three separate streams.
"""
import numpy as np
import pytest
import torch

from block_sparse_attention_45_b200 import binding as bsa
from block_sparse_attention_45_b200 import synth

pytestmark = pytest.mark.gpu

CASES = {
    "tiny": (synth.WORKLOADS["tiny"], 1, "same"),
    "small_g5": (synth.WORKLOADS["small"], 5, "separate"),          # groups of 5, 5, 2
    "small_all": (synth.WORKLOADS["small"], 12, "separate"),        # one group
    "b2_g2": (synth.custom("b2_h3", batch=2, heads=3, head_dim=64, q_block=128, k_block=64,
                           text_len=100, num_frames=3, latent_h=10, latent_w=16, top_p=0.8,
                           seed=21), 2, "separate"),                 # per batch: groups of 2, 1
}


def _host(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).pin_memory()


@pytest.mark.parametrize("case", sorted(CASES))
def test_pipeline_matches_device_calls(case):
    w, hpg, mode = CASES[case]
    x = synth.generate(w)
    qh, kh, vh = _host(x["q"]), _host(x["k"]), _host(x["v"])
    qd, kd, vd = qh.cuda(), kh.cuda(), vh.cuda()
    tp = [float(w.top_p)] * w.heads
    ref = bsa.sparse_attention(w, qd, kd, vd, tp, w.flags)
    torch.cuda.synchronize()

    B, H = w.batch, w.heads
    Cq = w.seq_pad // w.q_block
    ent = torch.full((B, H), float("nan"), dtype=torch.float32).pin_memory()
    entn = torch.full((B, H), float("nan"), dtype=torch.float32).pin_memory()
    cnt = torch.full((B, H, Cq), -7, dtype=torch.int32).pin_memory()
    err = torch.full((1,), -1, dtype=torch.int32).pin_memory()
    out = torch.full(qh.shape, 3.0, dtype=torch.bfloat16).pin_memory()
    extra = {}
    if mode == "separate":
        extra = dict(h2d_stream=torch.cuda.Stream(), d2h_stream=torch.cuda.Stream())
    stream = torch.cuda.Stream()
    res = bsa.sparse_attention_host(w, qh, kh, vh, tp, w.flags, heads_per_group=hpg, out=out,
                                    entropy=ent, entropy_norm=entn, kv_count=cnt, err_flag=err,
                                    stream=stream, **extra)
    stream.synchronize()
    assert res["out"] is out
    assert torch.equal(out, ref["out"].cpu())
    assert torch.equal(cnt, ref["kv_count"].cpu())
    assert torch.equal(ent, ref["entropy"].cpu())
    assert torch.equal(entn, ref["entropy_norm"].cpu())
    assert err.item() == 0


def test_pipeline_twice_reuses_the_workspace():
    w = synth.WORKLOADS["small"]
    x = synth.generate(w)
    qh, kh, vh = _host(x["q"]), _host(x["k"]), _host(x["v"])
    tp = [float(w.top_p)] * w.heads
    first = bsa.sparse_attention_host(w, qh, kh, vh, tp, w.flags, heads_per_group=4)
    ws = first["workspace"]
    # the second call sees the first call's leftovers in the workspace
    second = bsa.sparse_attention_host(w, qh, kh, vh, tp, w.flags, heads_per_group=4, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(first["out"], second["out"])
