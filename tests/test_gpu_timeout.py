"""The attention kernel's bounded waits, made to run out (needs a B200).

Every pipeline wait of the attention kernel gives up after a limit (2 s by
default), after which the kernel waits for the copies and products it already
started, releases its tensor memory, reports BSA_DEVERR_TIMEOUT and returns, so
that the context stays usable.  A limit of a nanosecond, far below the latency
of the kernel's first load, makes the waits run out on purpose: the call must
return with the flag set, and the next call with the default limit, on the same
stream, must give the same output as one made before.  Nothing here faults or
hangs the GPU: the limit only shortens waits that already have one.
"""
import numpy as np
import pytest
import torch

from block_sparse_attention_45_b200 import binding as bsa
from block_sparse_attention_45_b200 import synth
from tests.gpu_util import to_dev

pytestmark = pytest.mark.gpu


def test_short_wait_limit_stops_attention_and_reports_it():
    # one head of the HunyuanVideo shape (931 query blocks, text + 33 frames of 45x80)
    w = synth.custom("hunyuan_1head", heads=1, head_dim=128, text_len=256, num_frames=33,
                     latent_h=45, latent_w=80, q_block=128, k_block=128, top_p=0.9, seed=4,
                     kind="clustered", sigma_mean=2.0)
    x = synth.generate(w)
    q, k, v = to_dev(x["q"]), to_dev(x["k"]), to_dev(x["v"])
    sel = bsa.sparse_attention(w, q, k, v, [0.9], w.flags)
    idx, cnt = sel["kv_index"], sel["kv_count"]
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ref, ref_lse = bsa.attention_fwd(w, q, k, v, idx, cnt, err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    try:
        bsa.set_wait_limit_ns(1)
        for _ in range(2):   # twice: the second launch starts from a clean slate too
            err.zero_()
            out, lse = bsa.attention_fwd(w, q, k, v, idx, cnt, err_flag=err)
            torch.cuda.synchronize()
            assert int(err.item()) & bsa.DEVERR_TIMEOUT, int(err.item())
    finally:
        bsa.set_wait_limit_ns(0)
    err.zero_()
    out, lse = bsa.attention_fwd(w, q, k, v, idx, cnt, err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert torch.equal(out, ref)
    assert torch.equal(torch.nan_to_num(lse, nan=7.0), torch.nan_to_num(ref_lse, nan=7.0))
    print("selected pairs: %d" % int(cnt.sum().item()))
