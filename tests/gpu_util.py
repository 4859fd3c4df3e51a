"""Shared helpers for the GPU parity tests (inputs, calibrated top-p, transfers)."""
import functools
import json
import os

import numpy as np
import torch

import oracle
from block_sparse_attention_45_b200 import synth

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def to_dev(u16):
    """Raw bf16 bits (numpy uint16) -> CUDA bf16 tensor with the same bytes."""
    return torch.from_numpy(np.ascontiguousarray(u16).view(np.int16)).cuda().view(torch.bfloat16)


def to_host_f32(t):
    return t.float().cpu().numpy()


@functools.lru_cache(maxsize=1)
def calibrated():
    return json.load(open(os.path.join(GOLDEN, "top_p_calibrated.json")))


def top_p_of(w):
    if w.top_p is not None:
        return [float(w.top_p)] * w.heads
    return [float(x) for x in calibrated()[w.name]["top_p"]]


@functools.lru_cache(maxsize=2)
def inputs(name):
    w = synth.WORKLOADS[name]
    return w, synth.generate(w)


@functools.lru_cache(maxsize=2)
def oracle_selection(name):
    w, x = inputs(name)
    return oracle.select(w.layout(), x["q"], x["k"], top_p_of(w), w.flags)


def sample_rows(w, n_random=3, seed=0):
    """Flat query-block ids to check at full size: frame-0, text, last (ragged), random."""
    cq = w.seq_pad // w.q_block
    L = w.layout()
    f0, f1 = oracle.frame0_qblocks(L)
    rng = np.random.default_rng(seed)
    rows = {0 * cq + f0, (w.heads - 1) * cq + cq - 1, (w.heads // 2) * cq + min(f1 + 1, cq - 1)}
    if w.text_len > 0:
        rows.add((w.heads // 3) * cq + 0)
    while len(rows) < 4 + n_random:
        rows.add(int(rng.integers(w.batch * w.heads * cq)))
    return np.array(sorted(rows), np.int64)
