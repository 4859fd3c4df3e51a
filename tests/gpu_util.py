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


def sample_rows(w, n_random=64, seed=0, frame0_head=0):
    """Flat query-block ids to check at full size: the first frame-0 block, a text
    block, the ragged last block, every frame-0 block of head `frame0_head` (None:
    skip), and n_random random blocks spread over every head (random block of
    head r mod B*H for r = 0 .. n_random-1)."""
    cq = w.seq_pad // w.q_block
    L = w.layout()
    f0, f1 = oracle.frame0_qblocks(L)
    rng = np.random.default_rng(seed)
    rows = {0 * cq + f0, (w.heads - 1) * cq + cq - 1, (w.heads // 2) * cq + min(f1 + 1, cq - 1)}
    if w.text_len > 0:
        rows.add((w.heads // 3) * cq + 0)
    if frame0_head is not None and f1 >= f0:
        rows.update(frame0_head * cq + i for i in range(f0, f1 + 1))
    bh = w.batch * w.heads
    want = min(len(rows) + n_random, bh * cq)   # a small workload has fewer blocks than asked for
    r = 0
    while len(rows) < want:
        rows.add(int((r % bh) * cq + rng.integers(cq)))
        r += 1
    return np.array(sorted(rows), np.int64)
