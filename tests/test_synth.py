"""The seeded input generator both sides consume, on the CPU: reproducible per
seed and per head, zero padding rows, bf16 rounding equal to torch's, and the
clustered recipe's structure (tokens sharing a frame and an 8 x 8 latent patch
share their mean)."""
import numpy as np
import torch

from block_sparse_attention_45_b200 import synth


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(5)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 10.0 ** rng.integers(-6, 6, 100000),
                        np.array([0.0, -0.0, 1.0, -1.0, 1.00390625, 1.01171875, 3.0e38, 1e-40],
                                 np.float32)]).astype(np.float32)
    ours = synth.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    back = synth.bf16_bits_to_f32(ours)
    assert np.array_equal(back, torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_generation_is_reproducible_and_per_head():
    w = synth.custom("rep", batch=2, heads=3, head_dim=64, text_len=10, num_frames=2, latent_h=8,
                     latent_w=12, q_block=64, k_block=64, seed=77, kind="clustered")
    a = synth.generate(w, workers=1)
    b = synth.generate(w, workers=4)
    for t in ("q", "k", "v"):
        assert a[t].dtype == np.uint16 and a[t].shape == (2, 3, w.seq_pad, 64)
        assert np.array_equal(a[t], b[t])
        assert (a[t][:, :, w.seq_len:] == 0).all()          # padding rows are zero
    one = synth.generate(w, heads=[2], batches=[1])
    for t in ("q", "k", "v"):
        assert np.array_equal(one[t][0, 0], a[t][1, 2])
    other = synth.generate(synth.custom("rep", batch=2, heads=3, head_dim=64, text_len=10,
                                        num_frames=2, latent_h=8, latent_w=12, q_block=64,
                                        k_block=64, seed=78, kind="clustered"))
    assert not np.array_equal(other["q"], a["q"])
    assert not np.array_equal(a["q"], a["k"])               # Q and K are independent draws


def test_clustered_tokens_share_frame_and_patch_means():
    w = synth.custom("cl", heads=1, head_dim=128, text_len=0, num_frames=3, latent_h=16,
                     latent_w=16, q_block=128, k_block=128, seed=3, kind="clustered",
                     sigma_noise=0.05, sigma_mean=1.0)
    q = synth.bf16_bits_to_f32(synth.generate(w, tensors=("q",))["q"])[0, 0, :w.seq_len]
    vis = q.reshape(3, 16, 16, 128)
    # same frame and patch: the means agree up to the small noise
    same = np.abs(vis[1, 0, 0] - vis[1, 7, 7]).mean()
    # another 8 x 8 patch of the same frame, or another frame: different means
    other_patch = np.abs(vis[1, 0, 0] - vis[1, 8, 8]).mean()
    other_frame = np.abs(vis[1, 0, 0] - vis[2, 0, 0]).mean()
    assert same < 0.1 < min(other_patch, other_frame)
