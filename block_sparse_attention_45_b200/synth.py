"""Seeded synthetic video-DiT attention inputs (shared by the tests, the bench and smoke).

This module only draws random numbers and lays them out.  It holds none of the
method's arithmetic, so both the CUDA path and the CPU oracle may consume its
output.  Every tensor is returned as raw bf16 bit patterns (numpy uint16,
[B, H, seq_pad, D]); rows seq_len..seq_pad-1 are zero.

Token order follows "Attention matrix view: make only frame-0 query rows
dense" s1: [text tokens] + [frame 0 tokens] + [frame 1 tokens] + ..., each
frame a latent_h x latent_w grid flattened row-major.

The real workloads the pages measure on (Wan2.1, HunyuanVideo activations on
VBench prompts) are not available; these generators stand in for them with the
same shapes:
  * "tiny": Q, K, V = N(0,1) + a mean vector per 64-token block drawn from
    N(0, 1.5^2 I), independently for Q, K and V.
  * "clustered": for X in {Q, K} (independent draws), a visual token at frame f,
    latent row y, column x is N(0, s_n^2) + F_X[f] + G_X[y // 8, x // 8]
    (a per-frame mean and a mean per 8x8 latent patch, both N(0, s_m^2 I));
    a text token t is N(0, s_n^2) + T_X[t] with T_X[t] ~ N(0, s_m^2 I);
    V = N(0, 1).
Each (tensor, b, h) uses its own numpy PCG64 stream seeded with
[seed, tensor, b, h], so any head can be generated on its own.
"""
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, asdict

import numpy as np

TENSOR_IDS = {"q": 0, "k": 1, "v": 2}


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    heads: int
    head_dim: int
    text_len: int
    num_frames: int
    latent_h: int
    latent_w: int
    q_block: int
    k_block: int
    seed: int
    kind: str                 # "tiny" or "clustered"
    sigma_noise: float = 1.0
    sigma_mean: float = 1.5
    top_p: float = None       # fixed p for every head, or None when calibrated
    target_skip: float = None  # skipped-block fraction the per-head p is calibrated to
    text_keep: bool = True
    frame0_dense: bool = True
    pad_to: int = 128

    @property
    def tokens_per_frame(self):
        return self.latent_h * self.latent_w

    @property
    def seq_len(self):
        return self.text_len + self.num_frames * self.tokens_per_frame

    @property
    def seq_pad(self):
        m = max(self.pad_to, self.q_block, self.k_block)
        return -(-self.seq_len // m) * m

    def layout(self):
        """Geometry fields shared by the C ABI and the oracle."""
        return dict(batch=self.batch, heads=self.heads, seq_len=self.seq_len,
                    seq_pad=self.seq_pad, head_dim=self.head_dim, q_block=self.q_block,
                    k_block=self.k_block, text_len=self.text_len,
                    tokens_per_frame=self.tokens_per_frame, num_frames=self.num_frames)

    @property
    def flags(self):
        return (1 if self.text_keep else 0) | (2 if self.frame0_dense else 0)

    def describe(self):
        d = asdict(self)
        d.update(seq_len=self.seq_len, seq_pad=self.seq_pad)
        return d


# The five workload shapes (batch, heads, head_dim, token layout, block sizes,
# top-p policy, value distributions) used for parity and measurement.
WORKLOADS = {
    "tiny": Workload("tiny", batch=1, heads=2, head_dim=64, text_len=64, num_frames=2,
                     latent_h=8, latent_w=16, q_block=64, k_block=64, seed=0, kind="tiny",
                     sigma_mean=1.5, top_p=0.7, pad_to=64),
    "small": Workload("small", batch=1, heads=12, head_dim=128, text_len=512, num_frames=5,
                      latent_h=30, latent_w=52, q_block=128, k_block=128, seed=1,
                      kind="clustered", sigma_mean=1.5, top_p=0.9),
    "wan1.3b": Workload("wan1.3b", batch=1, heads=12, head_dim=128, text_len=0, num_frames=21,
                        latent_h=30, latent_w=52, q_block=128, k_block=128, seed=2,
                        kind="clustered", sigma_mean=2.0, target_skip=0.90),
    "wan14b": Workload("wan14b", batch=1, heads=40, head_dim=128, text_len=0, num_frames=21,
                       latent_h=30, latent_w=52, q_block=128, k_block=64, seed=3,
                       kind="clustered", sigma_mean=2.0, target_skip=0.92),
    "hunyuan": Workload("hunyuan", batch=1, heads=24, head_dim=128, text_len=256, num_frames=33,
                        latent_h=45, latent_w=80, q_block=128, k_block=128, seed=4,
                        kind="clustered", sigma_mean=2.0, target_skip=0.90),
}


# Key windows of autoregressive generation for head profiling ("Efficient
# Autoregressive Video Diffusion with Dummy Head", Step 0): a sink frame, a
# neighbor window and the current frame, 832x480 video (30x52 latent tokens per
# frame after 8x VAE and 2x2 patches), Wan2.1-1.3B heads.
WINDOWS = {
    "selfforcing": Workload("selfforcing", batch=1, heads=12, head_dim=128, text_len=0,
                            num_frames=5, latent_h=30, latent_w=52, q_block=128, k_block=128,
                            seed=5, kind="clustered", sigma_mean=2.0, top_p=0.9, text_keep=False,
                            frame0_dense=False),
}


def custom(name="custom", **kw):
    """A workload with explicit fields (edge-case parity tests)."""
    base = dict(batch=1, heads=1, head_dim=128, text_len=0, num_frames=1, latent_h=8,
                latent_w=16, q_block=128, k_block=128, seed=123, kind="tiny")
    base.update(kw)
    return Workload(name, **base)


def f32_to_bf16_bits(x):
    """Round-to-nearest-even fp32 -> bf16 bit patterns (inputs are finite)."""
    u = np.ascontiguousarray(x, np.float32).view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(h):
    return (np.asarray(h, np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _rng(w, tensor, b, h):
    return np.random.default_rng([w.seed, TENSOR_IDS[tensor], b, h])


def _draw_head(w, tensor, b, h):
    """fp32 [seq_len, D] values of one (tensor, batch, head)."""
    rng = _rng(w, tensor, b, h)
    S, D = w.seq_len, w.head_dim
    if w.kind == "tiny":
        nblk = -(-S // 64)
        means = (w.sigma_mean * rng.standard_normal((nblk, D), dtype=np.float32))
        x = w.sigma_noise * rng.standard_normal((S, D), dtype=np.float32)
        x += np.repeat(means, 64, axis=0)[:S]
        return x
    if w.kind != "clustered":
        raise ValueError(w.kind)
    if tensor == "v":
        return rng.standard_normal((S, D), dtype=np.float32)
    sm = np.float32(w.sigma_mean)
    T = sm * rng.standard_normal((w.text_len, D), dtype=np.float32)
    F = sm * rng.standard_normal((w.num_frames, D), dtype=np.float32)
    ph, pw = -(-w.latent_h // 8), -(-w.latent_w // 8)
    G = sm * rng.standard_normal((ph, pw, D), dtype=np.float32)
    x = np.float32(w.sigma_noise) * rng.standard_normal((S, D), dtype=np.float32)
    x[:w.text_len] += T
    Gx = np.repeat(np.repeat(G, 8, axis=0)[:w.latent_h], 8, axis=1)[:, :w.latent_w]
    mean = F[:, None, None, :] + Gx[None, :, :, :]
    vis = x[w.text_len:].reshape(w.num_frames, w.latent_h, w.latent_w, D)
    vis += mean
    return x


def generate(w, tensors=("q", "k", "v"), heads=None, batches=None, workers=None):
    """Raw bf16 bits, dict tensor -> uint16 [len(batches), len(heads), seq_pad, D].

    Every (tensor, b, h) has its own stream, so the result does not depend on
    `workers` (threads that fill different heads at the same time).
    """
    heads = list(range(w.heads)) if heads is None else list(heads)
    batches = list(range(w.batch)) if batches is None else list(batches)
    out = {t: np.zeros((len(batches), len(heads), w.seq_pad, w.head_dim), np.uint16)
           for t in tensors}
    jobs = [(t, bi, b, hi, h) for t in tensors for bi, b in enumerate(batches)
            for hi, h in enumerate(heads)]

    def fill(job):
        t, bi, b, hi, h = job
        out[t][bi, hi, :w.seq_len] = f32_to_bf16_bits(_draw_head(w, t, b, h))

    if workers is None:
        workers = min(len(jobs), max(1, (os.cpu_count() or 1)))
    if workers <= 1 or len(jobs) <= 1:
        for j in jobs:
            fill(j)
    else:
        with ThreadPoolExecutor(max_workers=workers) as ex:
            list(ex.map(fill, jobs))
    return out
