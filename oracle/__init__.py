"""CPU oracle for dynamic block-sparse attention -- TEST INFRASTRUCTURE ONLY.

Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline/reference legs
may import this package.  It wraps the plain fp64 C oracle (bsa_oracle.c) with
numpy marshalling and shares no code with the CUDA library.

Parity pins (tests/test_oracle_pins.py) hold every function here to closed
forms, invariants, brute force and independent library routines.  The one
reading that no pin can fix is recorded as "parity unpinned": the exact form of
P' and of the top-p rule beyond the prose of "Competition Domains Matter" s3
(its Eq. 1-3 are lost in the page text).
"""
import ctypes
import math
import os

import numpy as np

from . import build as _build

TEXT_KEEP = 1
FRAME0_DENSE = 2


class OracleLayout(ctypes.Structure):
    """Problem geometry, mirrored field by field from the caller's config."""
    _fields_ = [(n, ctypes.c_int32) for n in (
        "batch", "heads", "seq_len", "seq_pad", "head_dim", "q_block", "k_block",
        "text_len", "tokens_per_frame", "num_frames")]

    @classmethod
    def from_dict(cls, d):
        return cls(*[int(d[n]) for n, _ in cls._fields_])

    @property
    def cq(self):
        return self.seq_pad // self.q_block

    @property
    def ck(self):
        return self.seq_pad // self.k_block


class Oracle:
    """ctypes binding of one build of bsa_oracle.c (the default build, or a
    deliberately mutated copy used by the pin-sensitivity tests)."""

    def __init__(self, path=None):
        path = path or _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.POINTER
        lp = P(OracleLayout)
        vp = ctypes.c_void_p
        L.ora_block_count.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int]
        L.ora_block_count.restype = ctypes.c_int
        L.ora_frame0_qblocks.argtypes = [lp, P(ctypes.c_int), P(ctypes.c_int)]
        L.ora_text_kblocks.argtypes = [lp]
        L.ora_text_kblocks.restype = ctypes.c_int
        L.ora_pool.argtypes = [lp, vp, ctypes.c_int, vp]
        L.ora_scores.argtypes = [lp, vp, vp, vp]
        L.ora_entropy.argtypes = [lp, vp, ctypes.c_double, vp, vp]
        L.ora_topp.argtypes = [lp, vp, vp, vp, vp]
        L.ora_overrides.argtypes = [lp, ctypes.c_uint32, vp]
        L.ora_lists.argtypes = [lp, vp, vp, vp]
        L.ora_attention.argtypes = [lp, vp, vp, vp, vp, vp, ctypes.c_double, ctypes.c_long,
                                    vp, vp, vp]
        L.ora_value_norms.argtypes = [lp, vp, vp]
        L.ora_eg_route.argtypes = [lp, vp, vp]
        L.ora_eg_select.argtypes = [lp, vp, vp, vp, ctypes.c_float, vp, vp]
        L.ora_splitmix64.argtypes = [ctypes.c_uint64, ctypes.c_uint64]
        L.ora_splitmix64.restype = ctypes.c_uint64
        L.ora_inclusion.argtypes = [lp, vp, ctypes.c_float, ctypes.c_uint32, vp, vp]
        L.ora_sample_select.argtypes = [lp, vp, ctypes.c_float, ctypes.c_uint64, ctypes.c_uint32,
                                        vp, vp]
        L.ora_subclusters.argtypes = [lp, vp, ctypes.c_int, ctypes.c_int, vp, vp]
        L.ora_scores_clustered.argtypes = [lp, vp, vp, ctypes.c_int, vp, vp]
        L.ora_frame_scores.argtypes = [lp, vp, vp, ctypes.c_double, ctypes.c_int, vp]
        L.ora_dhp.argtypes = [vp, ctypes.c_int, ctypes.c_int, vp]
        L.ora_centroid_distortion.argtypes = [lp, vp, vp, vp, vp]
        L.ora_pool_select.argtypes = [lp, vp, vp, vp, ctypes.c_float, vp, ctypes.c_int, vp]
        L.ora_domain_route.argtypes = [lp, vp, ctypes.c_int, vp]
        L.ora_domain_route.restype = ctypes.c_int
        L.ora_num_threads.restype = ctypes.c_int
        self.lib = L

    def num_threads(self):
        return self.lib.ora_num_threads()

    def block_count(self, seq_len, block, idx):
        return self.lib.ora_block_count(seq_len, block, idx)

    def frame0_qblocks(self, L):
        L = _layout(L)
        a, b = ctypes.c_int(), ctypes.c_int()
        self.lib.ora_frame0_qblocks(ctypes.byref(L), ctypes.byref(a), ctypes.byref(b))
        return a.value, b.value

    def text_kblocks(self, L):
        L = _layout(L)
        return self.lib.ora_text_kblocks(ctypes.byref(L))

    def pool(self, L, x, block):
        """Block centroids, fp32 [B,H,C,D]."""
        L = _layout(L)
        x = _u16(x)
        out = np.empty((L.batch, L.heads, L.seq_pad // block, L.head_dim), np.float32)
        self.lib.ora_pool(ctypes.byref(L), _ptr(x), block, _ptr(out))
        return out

    def scores(self, L, qc, kc):
        """Cluster-size-weighted softmax P', fp32 [B,H,C_q,C_k]."""
        L = _layout(L)
        qc = np.ascontiguousarray(qc, np.float32)
        kc = np.ascontiguousarray(kc, np.float32)
        out = np.empty((L.batch, L.heads, L.cq, L.ck), np.float32)
        self.lib.ora_scores(ctypes.byref(L), _ptr(qc), _ptr(kc), _ptr(out))
        return out

    def subclusters(self, L, q, nsub, iters):
        """k-means sub-clusters of every query block: centroids fp32 [B,H,C_q,nsub,D] and
        sizes int32 [B,H,C_q,nsub]."""
        L = _layout(L)
        q = _u16(q)
        cent = np.empty((L.batch, L.heads, L.cq, nsub, L.head_dim), np.float32)
        size = np.empty((L.batch, L.heads, L.cq, nsub), np.int32)
        self.lib.ora_subclusters(ctypes.byref(L), _ptr(q), int(nsub), int(iters), _ptr(cent),
                                 _ptr(size))
        return cent, size

    def scores_clustered(self, L, cent, size, kc):
        """Block scores as the size-weighted mixture of the sub-centroid rows, fp32
        [B,H,C_q,C_k]."""
        L = _layout(L)
        cent = np.ascontiguousarray(cent, np.float32)
        size = np.ascontiguousarray(size, np.int32)
        kc = np.ascontiguousarray(kc, np.float32)
        out = np.empty((L.batch, L.heads, L.cq, L.ck), np.float32)
        self.lib.ora_scores_clustered(ctypes.byref(L), _ptr(cent), _ptr(size), int(cent.shape[3]),
                                      _ptr(kc), _ptr(out))
        return out

    def entropy(self, L, probs, eps=1e-8):
        """Per-head entropy and entropy / ln C_k, fp64 [B,H] each."""
        L = _layout(L)
        probs = np.ascontiguousarray(probs, np.float32)
        H = np.empty((L.batch, L.heads), np.float64)
        Hn = np.empty((L.batch, L.heads), np.float64)
        self.lib.ora_entropy(ctypes.byref(L), _ptr(probs), float(eps), _ptr(H), _ptr(Hn))
        return H, Hn

    def topp(self, L, probs, top_p):
        """Per-row top-p block mask (u8 [B,H,C_q,C_k]) and k* per row (int32 [B,H,C_q])."""
        L = _layout(L)
        probs = np.ascontiguousarray(probs, np.float32)
        tp = np.ascontiguousarray(np.broadcast_to(np.asarray(top_p, np.float32), (L.heads,)))
        mask = np.empty((L.batch, L.heads, L.cq, L.ck), np.uint8)
        kstar = np.empty((L.batch, L.heads, L.cq), np.int32)
        self.lib.ora_topp(ctypes.byref(L), _ptr(probs), _ptr(tp), _ptr(mask), _ptr(kstar))
        return mask, kstar

    def overrides(self, L, flags, mask):
        """Text-keep and frame-0-dense overrides applied to a copy of mask."""
        L = _layout(L)
        m = np.ascontiguousarray(mask, np.uint8).copy()
        self.lib.ora_overrides(ctypes.byref(L), int(flags), _ptr(m))
        return m

    def lists(self, L, mask):
        """Ascending selected key blocks per query block (-1 padded) and their counts."""
        L = _layout(L)
        mask = np.ascontiguousarray(mask, np.uint8)
        idx = np.empty((L.batch, L.heads, L.cq, L.ck), np.int32)
        cnt = np.empty((L.batch, L.heads, L.cq), np.int32)
        self.lib.ora_lists(ctypes.byref(L), _ptr(mask), _ptr(idx), _ptr(cnt))
        return idx, cnt

    def attention(self, L, q, k, v, mask=None, scale=None, rows=None, weight=None):
        """Exact softmax attention over the selected blocks (mask None = dense).

        rows: optional flat query-block ids (b*H*C_q + h*C_q + i).  Returns
        out fp32 [nrows, q_block, D] and lse fp32 [nrows, q_block]; with rows
        None the leading axis covers every query block in (b, h, i) order.
        weight: optional fp32 [B,H,C_q,C_k], multiplying every exp term of a
        key of block j (numerator and sum) by weight[b,h,i,j].
        """
        L = _layout(L)
        q, k, v = _u16(q), _u16(k), _u16(v)
        if scale is None:
            scale = 1.0 / math.sqrt(L.head_dim)
        m = None if mask is None else np.ascontiguousarray(mask, np.uint8)
        wt = None if weight is None else np.ascontiguousarray(weight, np.float32)
        if rows is None:
            n = L.batch * L.heads * L.cq
            r = None
        else:
            r = np.ascontiguousarray(rows, np.int64)
            n = r.shape[0]
        out = np.empty((n, L.q_block, L.head_dim), np.float32)
        lse = np.empty((n, L.q_block), np.float32)
        self.lib.ora_attention(ctypes.byref(L), _ptr(q), _ptr(k), _ptr(v), _ptr(m), _ptr(wt),
                               float(scale), n, _ptr(r), _ptr(out), _ptr(lse))
        return out, lse

    def frame_scores(self, L, q, k, scale=None, query_stride=1):
        """Per-head frame attention scores [alpha_sink, alpha_neighbor, alpha_current] of the
        current frame's queries, fp64 [B,H,3]."""
        L = _layout(L)
        q, k = _u16(q), _u16(k)
        if scale is None:
            scale = 1.0 / math.sqrt(L.head_dim)
        alpha = np.empty((L.batch, L.heads, 3), np.float64)
        self.lib.ora_frame_scores(ctypes.byref(L), _ptr(q), _ptr(k), float(scale), int(query_stride),
                                  _ptr(alpha))
        return alpha

    def dhp(self, alpha, n_dummy):
        """Dynamic Head Programming labels (0 sink, 1 neighbor, 2 dummy) of the heads of alpha [H,3]."""
        a = np.ascontiguousarray(alpha, np.float64)
        H = a.shape[0]
        label = np.empty(H, np.int32)
        self.lib.ora_dhp(_ptr(a), H, int(n_dummy), _ptr(label))
        return label

    def splitmix64(self, seed, idx):
        """The idx-th output (from 0) of SplitMix64 started from state `seed`."""
        return int(self.lib.ora_splitmix64(int(seed) & (2**64 - 1), int(idx) & (2**64 - 1)))

    def inclusion(self, L, probs, budget, flags):
        """Inclusion probability pi and weight 1/pi (fp32 [B,H,C_q,C_k]) of every pair."""
        L = _layout(L)
        probs = np.ascontiguousarray(probs, np.float32)
        pi = np.empty(probs.shape, np.float32)
        w = np.empty(probs.shape, np.float32)
        self.lib.ora_inclusion(ctypes.byref(L), _ptr(probs), float(budget), int(flags), _ptr(pi),
                               _ptr(w))
        return pi, w

    def sample_select(self, L, probs, budget, seed, flags):
        """One draw of the importance sampler: mask u8 and weight fp32 [B,H,C_q,C_k]."""
        L = _layout(L)
        probs = np.ascontiguousarray(probs, np.float32)
        mask = np.empty(probs.shape, np.uint8)
        weight = np.empty(probs.shape, np.float32)
        self.lib.ora_sample_select(ctypes.byref(L), _ptr(probs), float(budget),
                                   int(seed) & (2**64 - 1), int(flags), _ptr(mask), _ptr(weight))
        return mask, weight

    def value_norms(self, L, v):
        """||c^V_{h,j}||_2 of the value centroids, fp32 [B,H,C_k]."""
        L = _layout(L)
        v = _u16(v)
        out = np.empty((L.batch, L.heads, L.ck), np.float32)
        self.lib.ora_value_norms(ctypes.byref(L), _ptr(v), _ptr(out))
        return out

    def centroid_distortion(self, L, probs, vcent, mask):
        """Relative Frobenius error of the masked, row-renormalised centroid output
        against the dense one, per head, fp64 [B,H]."""
        L = _layout(L)
        probs = np.ascontiguousarray(probs, np.float32)
        vcent = np.ascontiguousarray(vcent, np.float32)
        mask = np.ascontiguousarray(mask, np.uint8)
        out = np.empty((L.batch, L.heads), np.float64)
        self.lib.ora_centroid_distortion(ctypes.byref(L), _ptr(probs), _ptr(vcent), _ptr(mask),
                                         _ptr(out))
        return out

    def eg_route(self, L, H):
        """Median split per batch entry: u8 [B,H], 1 for the floor(H/2) lowest-entropy heads."""
        L = _layout(L)
        H = np.ascontiguousarray(H, np.float64)
        low = np.empty((L.batch, L.heads), np.uint8)
        self.lib.ora_eg_route(ctypes.byref(L), _ptr(H), _ptr(low))
        return low

    def eg_select(self, L, probs, vnorm, top_p, pool_p, low):
        """Entropy-guided selection mask u8 [B,H,C_q,C_k] (no overrides): per-row top-p for
        the heads with low == 0, one cross-head pool per batch entry for the others.
        vnorm None ranks the pool by P' alone."""
        L = _layout(L)
        probs = np.ascontiguousarray(probs, np.float32)
        vn = None if vnorm is None else np.ascontiguousarray(vnorm, np.float32)
        tp = np.ascontiguousarray(np.broadcast_to(np.asarray(top_p, np.float32), (L.heads,)))
        low = np.ascontiguousarray(low, np.uint8)
        mask = np.empty((L.batch, L.heads, L.cq, L.ck), np.uint8)
        self.lib.ora_eg_select(ctypes.byref(L), _ptr(probs), _ptr(vn), _ptr(tp), float(pool_p),
                               _ptr(low), _ptr(mask))
        return mask

    def domain_route(self, L, H, domain):
        """Pools of the competition domain (0 per-row, 1 per-head, 2 grouped, 3 all-head,
        4 EG-Sparse): pool_of int8 [B,H] (-1 = per-row) and G, the pools per batch entry."""
        L = _layout(L)
        H = np.ascontiguousarray(H, np.float64)
        pool_of = np.empty((L.batch, L.heads), np.int8)
        G = self.lib.ora_domain_route(ctypes.byref(L), _ptr(H), int(domain), _ptr(pool_of))
        return pool_of, int(G)

    def pool_select(self, L, probs, vnorm, top_p, pool_p, pool_of, G):
        """Pooled top-p over the pools of pool_of (-1 heads per-row), u8 [B,H,C_q,C_k]."""
        L = _layout(L)
        probs = np.ascontiguousarray(probs, np.float32)
        vn = None if vnorm is None else np.ascontiguousarray(vnorm, np.float32)
        tp = np.ascontiguousarray(np.broadcast_to(np.asarray(top_p, np.float32), (L.heads,)))
        po = np.ascontiguousarray(pool_of, np.int8)
        mask = np.empty((L.batch, L.heads, L.cq, L.ck), np.uint8)
        self.lib.ora_pool_select(ctypes.byref(L), _ptr(probs), _ptr(vn), _ptr(tp), float(pool_p),
                                 _ptr(po), int(G), _ptr(mask))
        return mask

    def eg_selection(self, L, q, k, v, top_p, pool_p, flags, eps=1e-8, value_aware=True):
        """The entropy-guided selection stage: centroids, P', entropy, median split,
        per-row / pooled top-p with the safeguard, overrides, lists."""
        L = _layout(L)
        qc = self.pool(L, q, L.q_block)
        kc = self.pool(L, k, L.k_block)
        probs = self.scores(L, qc, kc)
        H, Hn = self.entropy(L, probs, eps)
        low = self.eg_route(L, H)
        vn = self.value_norms(L, v) if value_aware else None
        smask = self.eg_select(L, probs, vn, top_p, pool_p, low)
        m = self.overrides(L, flags, smask)
        idx, cnt = self.lists(L, m)
        return dict(probs=probs, entropy=H, entropy_norm=Hn, low=low, vnorm=vn, sel_mask=smask,
                    mask=m, kv_index=idx, kv_count=cnt)

    def select(self, L, q, k, top_p, flags, eps=1e-8):
        """The whole selection stage: centroids, P', entropy, top-p, overrides, lists."""
        L = _layout(L)
        qc = self.pool(L, q, L.q_block)
        kc = self.pool(L, k, L.k_block)
        probs = self.scores(L, qc, kc)
        H, Hn = self.entropy(L, probs, eps)
        tmask, kstar = self.topp(L, probs, top_p)
        m = self.overrides(L, flags, tmask)
        idx, cnt = self.lists(L, m)
        return dict(q_centroids=qc, k_centroids=kc, probs=probs, entropy=H, entropy_norm=Hn,
                    topp_mask=tmask, mask=m, kstar=kstar, kv_index=idx, kv_count=cnt)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _u16(x):
    x = np.ascontiguousarray(x)
    if x.dtype != np.uint16:
        raise TypeError("oracle inputs are raw bf16 bit patterns (uint16)")
    return x


def _layout(L):
    return L if isinstance(L, OracleLayout) else OracleLayout.from_dict(L)


_DEFAULT = None


def default():
    """The oracle built from bsa_oracle.c as committed."""
    global _DEFAULT
    if _DEFAULT is None:
        _DEFAULT = Oracle()
    return _DEFAULT


def __getattr__(name):
    # module-level shortcuts: oracle.pool(...), oracle.scores(...), ...
    if name in ("num_threads", "block_count", "frame0_qblocks", "text_kblocks", "pool",
                "scores", "entropy", "topp", "overrides", "lists", "attention", "select"):
        return getattr(default(), name)
    raise AttributeError(name)
