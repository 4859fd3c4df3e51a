"""Head profiling (frame attention scores) against the oracle (needs a B200).

"Efficient Autoregressive Video Diffusion with Dummy Head", Step 0: per head,
the current frame's attention mass on the sink frame, the neighbor window and
the current frame.  The GPU computes it as attention over a one-hot V with
bf16 probabilities, so alpha must match the fp64 oracle within 5e-3; the DHP
labels from the GPU's alpha must equal the oracle's wherever the decisions are
not closer than that.
"""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_45_b200 import binding as bsa
from block_sparse_attention_45_b200 import synth

pytestmark = pytest.mark.gpu

ALPHA_ABS = 5e-3

WINDOWS = {
    "f5_d128": synth.custom("f5_d128", heads=4, head_dim=128, num_frames=5, latent_h=10,
                            latent_w=20, q_block=128, k_block=128, seed=41, kind="clustered",
                            sigma_mean=2.0),
    "f3_d64_ragged": synth.custom("f3_d64_ragged", heads=3, head_dim=64, num_frames=3, latent_h=10,
                                  latent_w=16, q_block=64, k_block=128, seed=42, kind="clustered",
                                  sigma_mean=2.0),
    "f2_b2": synth.custom("f2_b2", batch=2, heads=2, head_dim=64, num_frames=2, latent_h=10,
                          latent_w=17, q_block=128, k_block=64, seed=43, kind="clustered"),
    "selfforcing": synth.WINDOWS["selfforcing"],
}


def _dev_bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)


@pytest.mark.parametrize("stride", [1, 7])
@pytest.mark.parametrize("name", sorted(WINDOWS))
def test_frame_scores_match_the_oracle(name, stride):
    w = WINDOWS[name]
    x = synth.generate(w)
    ora = oracle.default()
    a_o = ora.frame_scores(w.layout(), x["q"], x["k"], query_stride=stride)
    a_g = bsa.frame_scores(w, _dev_bf16(x["q"]), _dev_bf16(x["k"]), query_stride=stride)
    torch.cuda.synchronize()
    a_g = a_g.cpu().numpy().astype(np.float64)
    assert np.abs(a_g - a_o).max() <= ALPHA_ABS, np.abs(a_g - a_o).max()
    np.testing.assert_allclose(a_g.sum(-1), 1.0, atol=ALPHA_ABS)
    if w.num_frames == 2:
        assert (a_g[..., 1] == 0).all()
    # labels: equal wherever no decision is within the tolerance
    H = w.heads
    for b in range(w.batch):
        for n_dummy in range(H + 1):
            lab_g = bsa.dhp_labels(a_g[b].astype(np.float32), n_dummy)
            lab_o = ora.dhp(a_o[b], n_dummy)
            lv = np.maximum(a_o[b, :, 0], a_o[b, :, 1])
            srt = np.sort(lv)
            cut_gap = np.inf if n_dummy in (0, H) else srt[n_dummy] - srt[n_dummy - 1]
            role_gap = np.abs(a_o[b, :, 0] - a_o[b, :, 1])
            if cut_gap > 2 * ALPHA_ABS:
                assert np.array_equal(lab_g == 2, lab_o == 2), (b, n_dummy)
                firm = (lab_o != 2) & (role_gap > 2 * ALPHA_ABS)
                assert np.array_equal(lab_g[firm], lab_o[firm]), (b, n_dummy)


def test_zero_queries_give_the_group_sizes():
    """Q = 0: every query attends uniformly, alpha = (1, F - 2, 1) / F exactly up to bf16 P."""
    w = WINDOWS["f5_d128"]
    x = synth.generate(w)
    q = torch.zeros((w.batch, w.heads, w.seq_pad, w.head_dim), dtype=torch.bfloat16, device="cuda")
    a = bsa.frame_scores(w, q, _dev_bf16(x["k"]))
    torch.cuda.synchronize()
    F = w.num_frames
    np.testing.assert_allclose(a.cpu().numpy(), np.broadcast_to([1 / F, (F - 2) / F, 1 / F], a.shape),
                               atol=2e-3)
