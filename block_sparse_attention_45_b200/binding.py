"""ctypes binding of libbsa.so (include/bsa.h): argument marshalling only.

Every step of the computation runs in the CUDA kernels behind the C ABI; this
module only checks tensor metadata, allocates outputs with torch (device
memory is plumbing) and passes raw pointers plus the current CUDA stream.
There is no CPU fallback: if the library is missing, every call raises.
"""
import ctypes
import math
import os
import re

import numpy as np
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libbsa.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "bsa.h")

BSA_OK = 0
BSA_ERR_INVALID_ARG = 1
BSA_ERR_UNSUPPORTED = 2
BSA_ERR_LAUNCH = 3
BSA_ERR_DRIVER = 4
TEXT_KEEP = 1
FRAME0_DENSE = 2
DEVERR_BAD_INDEX = 1
DEVERR_BAD_COUNT = 2
DEVERR_TIMEOUT = 4

LAYOUT_FIELDS = ("batch", "heads", "seq_len", "seq_pad", "head_dim", "q_block", "k_block",
                 "text_len", "tokens_per_frame", "num_frames")


class BsaLayout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in LAYOUT_FIELDS]


class BsaError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        super().__init__("%s failed: %s" % (fn, status_string(status)))


_LIB = None


def load():
    """Load libbsa.so (raises if it was not built)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("libbsa.so is not built; run `python -m block_sparse_attention_45_b200.build` "
                               "(there is no CPU fallback)")
        L = ctypes.CDLL(LIB_PATH)
        lp = ctypes.POINTER(BsaLayout)
        vp = ctypes.c_void_p
        L.bsa_block_scores.argtypes = [lp, vp, vp, vp, vp, vp, vp]
        L.bsa_block_scores.restype = ctypes.c_int
        L.bsa_build_mask_workspace_bytes.argtypes = [lp]
        L.bsa_build_mask_workspace_bytes.restype = ctypes.c_size_t
        L.bsa_build_mask.argtypes = [lp, vp, vp, ctypes.c_uint32, ctypes.c_float, vp, vp, vp, vp,
                                     vp, vp, vp]
        L.bsa_build_mask.restype = ctypes.c_int
        L.bsa_build_mask_noalloc.argtypes = [lp, vp, vp, ctypes.c_uint32, ctypes.c_float, vp, vp,
                                             vp, vp, vp, vp]
        L.bsa_build_mask_noalloc.restype = ctypes.c_int
        L.bsa_attention_fwd.argtypes = [lp, vp, vp, vp, vp, vp, ctypes.c_float, vp, vp, vp, vp, vp]
        L.bsa_attention_fwd.restype = ctypes.c_int
        L.bsa_attention_workspace_bytes.argtypes = [lp]
        L.bsa_attention_workspace_bytes.restype = ctypes.c_size_t
        L.bsa_dense_fwd.argtypes = [lp, vp, vp, vp, ctypes.c_float, vp, vp, vp, vp, vp]
        L.bsa_dense_fwd.restype = ctypes.c_int
        L.bsa_sparse_attention_host.argtypes = [lp, ctypes.c_int, vp, vp, vp, vp, ctypes.c_uint32,
                                                ctypes.c_float, ctypes.c_float, vp, vp, vp, vp, vp,
                                                vp, ctypes.c_size_t, vp, vp, vp]
        L.bsa_sparse_attention_host.restype = ctypes.c_int
        L.bsa_pipeline_workspace_bytes.argtypes = [lp, ctypes.c_int]
        L.bsa_pipeline_workspace_bytes.restype = ctypes.c_size_t
        L.bsa_value_norms.argtypes = [lp, vp, vp, vp]
        L.bsa_value_norms.restype = ctypes.c_int
        L.bsa_build_mask_eg.argtypes = [lp, vp, vp, vp, ctypes.c_float, ctypes.c_uint32,
                                        ctypes.c_float, vp, vp, vp, vp, vp, vp, vp, vp]
        L.bsa_build_mask_eg.restype = ctypes.c_int
        L.bsa_block_scores_clustered.argtypes = [lp, vp, vp, ctypes.c_int, ctypes.c_int, vp, vp, vp,
                                                 vp, vp, vp]
        L.bsa_block_scores_clustered.restype = ctypes.c_int
        L.bsa_block_scores_clustered_workspace_bytes.argtypes = [lp, ctypes.c_int]
        L.bsa_block_scores_clustered_workspace_bytes.restype = ctypes.c_size_t
        L.bsa_frame_scores.argtypes = [lp, vp, vp, ctypes.c_float, ctypes.c_int, vp, vp, vp]
        L.bsa_frame_scores.restype = ctypes.c_int
        L.bsa_frame_scores_workspace_bytes.argtypes = [lp]
        L.bsa_frame_scores_workspace_bytes.restype = ctypes.c_size_t
        L.bsa_dhp_labels.argtypes = [vp, ctypes.c_int, ctypes.c_int, vp]
        L.bsa_dhp_labels.restype = ctypes.c_int
        L.bsa_build_mask_sampled.argtypes = [lp, vp, ctypes.c_float, ctypes.c_uint64, ctypes.c_uint32,
                                             vp, vp, vp, vp, vp]
        L.bsa_build_mask_sampled.restype = ctypes.c_int
        L.bsa_attention_fwd_weighted.argtypes = [lp, vp, vp, vp, vp, vp, vp, ctypes.c_float, vp, vp,
                                                 vp, vp, vp]
        L.bsa_attention_fwd_weighted.restype = ctypes.c_int
        L.bsa_build_mask_eg_workspace_bytes.argtypes = [lp]
        L.bsa_build_mask_eg_workspace_bytes.restype = ctypes.c_size_t
        L.bsa_build_mask_domain.argtypes = [lp, ctypes.c_int, vp, vp, vp, ctypes.c_float, ctypes.c_uint32,
                                            ctypes.c_float, vp, vp, vp, vp, vp, vp, vp, vp]
        L.bsa_build_mask_domain.restype = ctypes.c_int
        L.bsa_build_mask_domain_workspace_bytes.argtypes = [lp, ctypes.c_int]
        L.bsa_build_mask_domain_workspace_bytes.restype = ctypes.c_size_t
        L.bsa_status_string.argtypes = [ctypes.c_int]
        L.bsa_status_string.restype = ctypes.c_char_p
        L.bsa_version.argtypes = []
        L.bsa_version.restype = ctypes.c_int
        L.bsa_set_wait_limit_ns.argtypes = [ctypes.c_ulonglong]
        L.bsa_set_wait_limit_ns.restype = ctypes.c_int
        _LIB = L
    return _LIB


def declared_symbols():
    """Function names declared in include/bsa.h."""
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*(bsa_[a-z_0-9]+)\s*\(",
                                 text, re.M)))


def set_wait_limit_ns(ns):
    """bsa_set_wait_limit_ns: limit of the attention kernel's pipeline waits (0: default 2 s)."""
    _check("bsa_set_wait_limit_ns", load().bsa_set_wait_limit_ns(int(ns)))


def status_string(status):
    return load().bsa_status_string(int(status)).decode()


def make_layout(layout):
    if isinstance(layout, BsaLayout):
        return layout
    if hasattr(layout, "layout"):
        layout = layout.layout()
    return BsaLayout(*[int(layout[n]) for n in LAYOUT_FIELDS])


def _ptr(t):
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(fn, rc):
    if rc != BSA_OK:
        raise BsaError(fn, rc)


def _need(t, name, dtype, shape):
    if t.dtype != dtype:
        raise TypeError("%s: expected %s, got %s" % (name, dtype, t.dtype))
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if tuple(t.shape) != tuple(shape):
        raise ValueError("%s: expected shape %s, got %s" % (name, tuple(shape), tuple(t.shape)))


def dims(L):
    L = make_layout(L)
    return dict(B=L.batch, H=L.heads, S=L.seq_len, Sp=L.seq_pad, D=L.head_dim,
                Cq=L.seq_pad // L.q_block, Ck=L.seq_pad // L.k_block)


def block_scores(layout, q, k, q_centroids=None, k_centroids=None, probs=None, stream=None):
    """bsa_block_scores: returns (q_centroids, k_centroids, probs)."""
    L = make_layout(layout)
    d = dims(L)
    qkv = (d["B"], d["H"], d["Sp"], d["D"])
    _need(q, "q", torch.bfloat16, qkv)
    _need(k, "k", torch.bfloat16, qkv)
    dev = q.device
    if q_centroids is None:
        q_centroids = torch.empty((d["B"], d["H"], d["Cq"], d["D"]), dtype=torch.float32, device=dev)
    if k_centroids is None:
        k_centroids = torch.empty((d["B"], d["H"], d["Ck"], d["D"]), dtype=torch.float32, device=dev)
    if probs is None:
        probs = torch.empty((d["B"], d["H"], d["Cq"], d["Ck"]), dtype=torch.float32, device=dev)
    _need(q_centroids, "q_centroids", torch.float32, (d["B"], d["H"], d["Cq"], d["D"]))
    _need(k_centroids, "k_centroids", torch.float32, (d["B"], d["H"], d["Ck"], d["D"]))
    _need(probs, "probs", torch.float32, (d["B"], d["H"], d["Cq"], d["Ck"]))
    rc = load().bsa_block_scores(ctypes.byref(L), _ptr(q), _ptr(k), _ptr(q_centroids),
                                 _ptr(k_centroids), _ptr(probs), _stream(stream))
    _check("bsa_block_scores", rc)
    return q_centroids, k_centroids, probs


def workspace_bytes(layout):
    L = make_layout(layout)
    return int(load().bsa_build_mask_workspace_bytes(ctypes.byref(L)))


def build_mask(layout, probs, top_p, flags, eps=1e-8, mask=None, kv_index=None, kv_count=None,
               entropy=None, entropy_norm=None, workspace=None, with_mask=True,
               with_entropy=True, stream=None):
    """bsa_build_mask: returns dict(mask, kv_index, kv_count, entropy, entropy_norm)."""
    L = make_layout(layout)
    d = dims(L)
    _need(probs, "probs", torch.float32, (d["B"], d["H"], d["Cq"], d["Ck"]))
    dev = probs.device
    tp = (ctypes.c_float * d["H"])(*[float(x) for x in
                                     (list(top_p) if hasattr(top_p, "__len__") else [top_p] * d["H"])])
    if len(tp) != d["H"]:
        raise ValueError("top_p needs one value per head")
    if mask is None and with_mask:
        mask = torch.empty((d["B"], d["H"], d["Cq"], d["Ck"]), dtype=torch.uint8, device=dev)
    if kv_index is None:
        kv_index = torch.empty((d["B"], d["H"], d["Cq"], d["Ck"]), dtype=torch.int32, device=dev)
    if kv_count is None:
        kv_count = torch.empty((d["B"], d["H"], d["Cq"]), dtype=torch.int32, device=dev)
    if with_entropy:
        if entropy is None:
            entropy = torch.empty((d["B"], d["H"]), dtype=torch.float32, device=dev)
        if entropy_norm is None:
            entropy_norm = torch.empty((d["B"], d["H"]), dtype=torch.float32, device=dev)
        if workspace is None:
            workspace = torch.empty(workspace_bytes(L), dtype=torch.uint8, device=dev)
    rc = load().bsa_build_mask(ctypes.byref(L), _ptr(probs), ctypes.cast(tp, ctypes.c_void_p),
                               int(flags), float(eps), _ptr(mask), _ptr(kv_index), _ptr(kv_count),
                               _ptr(entropy), _ptr(entropy_norm), _ptr(workspace), _stream(stream))
    _check("bsa_build_mask", rc)
    return dict(mask=mask, kv_index=kv_index, kv_count=kv_count, entropy=entropy,
                entropy_norm=entropy_norm)


def value_norms(layout, v, vnorm=None, stream=None):
    """bsa_value_norms: ||c^V_{h,j}||_2 of the value centroids, fp32 [B,H,C_k]."""
    L = make_layout(layout)
    d = dims(L)
    _need(v, "v", torch.bfloat16, (d["B"], d["H"], L.seq_pad, L.head_dim))
    if vnorm is None:
        vnorm = torch.empty((d["B"], d["H"], d["Ck"]), dtype=torch.float32, device=v.device)
    _check("bsa_value_norms", load().bsa_value_norms(ctypes.byref(L), _ptr(v), _ptr(vnorm),
                                                     _stream(stream)))
    return vnorm


def eg_workspace_bytes(layout):
    L = make_layout(layout)
    return int(load().bsa_build_mask_eg_workspace_bytes(ctypes.byref(L)))


# Competition domains (enum bsa_domain).
DOMAIN_ROW, DOMAIN_HEAD, DOMAIN_GROUPED, DOMAIN_ALL, DOMAIN_EG = 0, 1, 2, 3, 4


def domain_workspace_bytes(layout, domain):
    L = make_layout(layout)
    return int(load().bsa_build_mask_domain_workspace_bytes(ctypes.byref(L), int(domain)))


def _pooled_outputs(d, dev, mask, kv_index, kv_count, entropy, entropy_norm, with_mask):
    if mask is None and with_mask:
        mask = torch.empty((d["B"], d["H"], d["Cq"], d["Ck"]), dtype=torch.uint8, device=dev)
    if kv_index is None:
        kv_index = torch.empty((d["B"], d["H"], d["Cq"], d["Ck"]), dtype=torch.int32, device=dev)
    if kv_count is None:
        kv_count = torch.empty((d["B"], d["H"], d["Cq"]), dtype=torch.int32, device=dev)
    if entropy is None:
        entropy = torch.empty((d["B"], d["H"]), dtype=torch.float32, device=dev)
    if entropy_norm is None:
        entropy_norm = torch.empty((d["B"], d["H"]), dtype=torch.float32, device=dev)
    _need(entropy, "entropy", torch.float32, (d["B"], d["H"]))
    _need(entropy_norm, "entropy_norm", torch.float32, (d["B"], d["H"]))
    return mask, kv_index, kv_count, entropy, entropy_norm


def _pooled_inputs(L, probs, vnorm, top_p):
    d = dims(L)
    _need(probs, "probs", torch.float32, (d["B"], d["H"], d["Cq"], d["Ck"]))
    if vnorm is not None:
        _need(vnorm, "vnorm", torch.float32, (d["B"], d["H"], d["Ck"]))
    vals = list(top_p) if hasattr(top_p, "__len__") else [top_p] * d["H"]
    if len(vals) != d["H"]:
        raise ValueError("top_p needs one value per head")
    return d, (ctypes.c_float * d["H"])(*[float(x) for x in vals])


def build_mask_eg(layout, probs, vnorm, top_p, pool_p, flags, eps=1e-8, mask=None,
                  kv_index=None, kv_count=None, workspace=None, with_mask=True, stream=None,
                  entropy=None, entropy_norm=None, low_heads=None):
    """bsa_build_mask_eg (entropy-guided grouped cross-head selection): returns
    dict(mask, kv_index, kv_count, entropy, entropy_norm, low_heads).  vnorm None
    ranks the pools by P' alone."""
    L = make_layout(layout)
    d, tp = _pooled_inputs(L, probs, vnorm, top_p)
    dev = probs.device
    mask, kv_index, kv_count, entropy, entropy_norm = _pooled_outputs(
        d, dev, mask, kv_index, kv_count, entropy, entropy_norm, with_mask)
    low = low_heads
    if low is None:
        low = torch.empty((d["B"], d["H"]), dtype=torch.uint8, device=dev)
    _need(low, "low_heads", torch.uint8, (d["B"], d["H"]))
    if workspace is None:
        workspace = torch.empty(eg_workspace_bytes(L), dtype=torch.uint8, device=dev)
    rc = load().bsa_build_mask_eg(ctypes.byref(L), _ptr(probs), _ptr(vnorm),
                                  ctypes.cast(tp, ctypes.c_void_p), float(pool_p), int(flags),
                                  float(eps), _ptr(mask), _ptr(kv_index), _ptr(kv_count),
                                  _ptr(entropy), _ptr(entropy_norm), _ptr(low), _ptr(workspace),
                                  _stream(stream))
    _check("bsa_build_mask_eg", rc)
    return dict(mask=mask, kv_index=kv_index, kv_count=kv_count, entropy=entropy,
                entropy_norm=entropy_norm, low_heads=low)


def build_mask_domain(layout, domain, probs, vnorm, top_p, pool_p, flags, eps=1e-8, mask=None,
                      kv_index=None, kv_count=None, workspace=None, with_mask=True, stream=None,
                      entropy=None, entropy_norm=None, pool_of=None):
    """bsa_build_mask_domain (pooled top-p over a competition domain, DOMAIN_*):
    returns dict(mask, kv_index, kv_count, entropy, entropy_norm, pool_of)."""
    L = make_layout(layout)
    d, tp = _pooled_inputs(L, probs, vnorm, top_p)
    dev = probs.device
    mask, kv_index, kv_count, entropy, entropy_norm = _pooled_outputs(
        d, dev, mask, kv_index, kv_count, entropy, entropy_norm, with_mask)
    if pool_of is None:
        pool_of = torch.empty((d["B"], d["H"]), dtype=torch.int8, device=dev)
    _need(pool_of, "pool_of", torch.int8, (d["B"], d["H"]))
    if workspace is None:
        n = domain_workspace_bytes(L, domain)
        if n == 0:
            raise BsaError("bsa_build_mask_domain", BSA_ERR_INVALID_ARG)
        workspace = torch.empty(n, dtype=torch.uint8, device=dev)
    rc = load().bsa_build_mask_domain(ctypes.byref(L), int(domain), _ptr(probs), _ptr(vnorm),
                                      ctypes.cast(tp, ctypes.c_void_p), float(pool_p), int(flags),
                                      float(eps), _ptr(mask), _ptr(kv_index), _ptr(kv_count),
                                      _ptr(entropy), _ptr(entropy_norm), _ptr(pool_of),
                                      _ptr(workspace), _stream(stream))
    _check("bsa_build_mask_domain", rc)
    return dict(mask=mask, kv_index=kv_index, kv_count=kv_count, entropy=entropy,
                entropy_norm=entropy_norm, pool_of=pool_of)


def attention_workspace_bytes(layout):
    L = make_layout(layout)
    return int(load().bsa_attention_workspace_bytes(ctypes.byref(L)))


def _attn_workspace(L, device, workspace):
    if workspace is None:
        workspace = torch.empty(attention_workspace_bytes(L), dtype=torch.uint8, device=device)
    return workspace


def attention_fwd(layout, q, k, v, kv_index, kv_count, softmax_scale=None, out=None, lse=None,
                  err_flag=None, with_lse=True, workspace=None, stream=None):
    """bsa_attention_fwd: returns (out, lse)."""
    L = make_layout(layout)
    d = dims(L)
    qkv = (d["B"], d["H"], d["Sp"], d["D"])
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, torch.bfloat16, qkv)
    _need(kv_index, "kv_index", torch.int32, (d["B"], d["H"], d["Cq"], d["Ck"]))
    _need(kv_count, "kv_count", torch.int32, (d["B"], d["H"], d["Cq"]))
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(d["D"])
    if out is None:
        out = torch.empty(qkv, dtype=torch.bfloat16, device=q.device)
    if lse is None and with_lse:
        lse = torch.empty((d["B"], d["H"], d["Sp"]), dtype=torch.float32, device=q.device)
    workspace = _attn_workspace(L, q.device, workspace)
    rc = load().bsa_attention_fwd(ctypes.byref(L), _ptr(q), _ptr(k), _ptr(v), _ptr(kv_index),
                                  _ptr(kv_count), float(softmax_scale), _ptr(out), _ptr(lse),
                                  _ptr(err_flag), _ptr(workspace), _stream(stream))
    _check("bsa_attention_fwd", rc)
    return out, lse


def clustered_workspace_bytes(layout, n_sub):
    L = make_layout(layout)
    return int(load().bsa_block_scores_clustered_workspace_bytes(ctypes.byref(L), int(n_sub)))


def block_scores_clustered(layout, q, k, n_sub, iters, sub_centroids=None, sub_sizes=None,
                           k_centroids=None, probs=None, workspace=None, stream=None):
    """bsa_block_scores_clustered: returns (sub_centroids, sub_sizes, k_centroids, probs)."""
    L = make_layout(layout)
    d = dims(L)
    qkv = (d["B"], d["H"], d["Sp"], d["D"])
    _need(q, "q", torch.bfloat16, qkv)
    _need(k, "k", torch.bfloat16, qkv)
    dev = q.device
    f32 = dict(dtype=torch.float32, device=dev)
    if sub_centroids is None:
        sub_centroids = torch.empty((d["B"], d["H"], d["Cq"], n_sub, d["D"]), **f32)
    if sub_sizes is None:
        sub_sizes = torch.empty((d["B"], d["H"], d["Cq"], n_sub), dtype=torch.int32, device=dev)
    if k_centroids is None:
        k_centroids = torch.empty((d["B"], d["H"], d["Ck"], d["D"]), **f32)
    if probs is None:
        probs = torch.empty((d["B"], d["H"], d["Cq"], d["Ck"]), **f32)
    if workspace is None:
        workspace = torch.empty(max(clustered_workspace_bytes(L, n_sub), 256), dtype=torch.uint8,
                                device=dev)
    rc = load().bsa_block_scores_clustered(ctypes.byref(L), _ptr(q), _ptr(k), int(n_sub), int(iters),
                                           _ptr(sub_centroids), _ptr(sub_sizes), _ptr(k_centroids),
                                           _ptr(probs), _ptr(workspace), _stream(stream))
    _check("bsa_block_scores_clustered", rc)
    return sub_centroids, sub_sizes, k_centroids, probs


HEAD_SINK, HEAD_NEIGHBOR, HEAD_DUMMY = 0, 1, 2


def frame_scores_workspace_bytes(layout):
    L = make_layout(layout)
    return int(load().bsa_frame_scores_workspace_bytes(ctypes.byref(L)))


def frame_scores(layout, q, k, softmax_scale=None, query_stride=1, alpha=None, workspace=None,
                 stream=None):
    """bsa_frame_scores: [alpha_sink, alpha_neighbor, alpha_current] per head, fp32 [B,H,3]."""
    L = make_layout(layout)
    d = dims(L)
    qkv = (d["B"], d["H"], d["Sp"], d["D"])
    _need(q, "q", torch.bfloat16, qkv)
    _need(k, "k", torch.bfloat16, qkv)
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(d["D"])
    if alpha is None:
        alpha = torch.empty((d["B"], d["H"], 3), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = torch.empty(frame_scores_workspace_bytes(L), dtype=torch.uint8, device=q.device)
    rc = load().bsa_frame_scores(ctypes.byref(L), _ptr(q), _ptr(k), float(softmax_scale),
                                 int(query_stride), _ptr(alpha), _ptr(workspace), _stream(stream))
    _check("bsa_frame_scores", rc)
    return alpha


def dhp_labels(alpha, n_dummy):
    """bsa_dhp_labels (host): labels 0 sink, 1 neighbor, 2 dummy of the heads of alpha [H, 3]."""
    a = np.ascontiguousarray(np.asarray(alpha, np.float32).reshape(-1, 3))
    labels = np.empty(a.shape[0], np.int32)
    rc = load().bsa_dhp_labels(a.ctypes.data_as(ctypes.c_void_p), a.shape[0], int(n_dummy),
                               labels.ctypes.data_as(ctypes.c_void_p))
    _check("bsa_dhp_labels", rc)
    return labels


def build_mask_sampled(layout, probs, budget, seed, flags, mask=None, kv_index=None,
                       kv_weight=None, kv_count=None, with_mask=True, stream=None):
    """bsa_build_mask_sampled (importance sampling with inverse-inclusion-probability
    weights): returns dict(mask, kv_index, kv_weight, kv_count)."""
    L = make_layout(layout)
    d = dims(L)
    _need(probs, "probs", torch.float32, (d["B"], d["H"], d["Cq"], d["Ck"]))
    dev = probs.device
    shp = (d["B"], d["H"], d["Cq"], d["Ck"])
    if mask is None and with_mask:
        mask = torch.empty(shp, dtype=torch.uint8, device=dev)
    if kv_index is None:
        kv_index = torch.empty(shp, dtype=torch.int32, device=dev)
    if kv_weight is None:
        kv_weight = torch.empty(shp, dtype=torch.float32, device=dev)
    if kv_count is None:
        kv_count = torch.empty((d["B"], d["H"], d["Cq"]), dtype=torch.int32, device=dev)
    _need(kv_index, "kv_index", torch.int32, shp)
    _need(kv_weight, "kv_weight", torch.float32, shp)
    _need(kv_count, "kv_count", torch.int32, (d["B"], d["H"], d["Cq"]))
    rc = load().bsa_build_mask_sampled(ctypes.byref(L), _ptr(probs), float(budget),
                                       int(seed) & (2**64 - 1), int(flags), _ptr(mask),
                                       _ptr(kv_index), _ptr(kv_weight), _ptr(kv_count),
                                       _stream(stream))
    _check("bsa_build_mask_sampled", rc)
    return dict(mask=mask, kv_index=kv_index, kv_weight=kv_weight, kv_count=kv_count)


def attention_fwd_weighted(layout, q, k, v, kv_index, kv_weight, kv_count, softmax_scale=None,
                           out=None, lse=None, err_flag=None, with_lse=True, workspace=None,
                           stream=None):
    """bsa_attention_fwd_weighted: returns (out, lse)."""
    L = make_layout(layout)
    d = dims(L)
    qkv = (d["B"], d["H"], d["Sp"], d["D"])
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, torch.bfloat16, qkv)
    _need(kv_index, "kv_index", torch.int32, (d["B"], d["H"], d["Cq"], d["Ck"]))
    _need(kv_weight, "kv_weight", torch.float32, (d["B"], d["H"], d["Cq"], d["Ck"]))
    _need(kv_count, "kv_count", torch.int32, (d["B"], d["H"], d["Cq"]))
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(d["D"])
    if out is None:
        out = torch.empty(qkv, dtype=torch.bfloat16, device=q.device)
    if lse is None and with_lse:
        lse = torch.empty((d["B"], d["H"], d["Sp"]), dtype=torch.float32, device=q.device)
    workspace = _attn_workspace(L, q.device, workspace)
    rc = load().bsa_attention_fwd_weighted(ctypes.byref(L), _ptr(q), _ptr(k), _ptr(v),
                                           _ptr(kv_index), _ptr(kv_weight), _ptr(kv_count),
                                           float(softmax_scale), _ptr(out), _ptr(lse),
                                           _ptr(err_flag), _ptr(workspace), _stream(stream))
    _check("bsa_attention_fwd_weighted", rc)
    return out, lse


def dense_fwd(layout, q, k, v, softmax_scale=None, out=None, lse=None, err_flag=None,
              with_lse=True, workspace=None, stream=None):
    """bsa_dense_fwd: returns (out, lse)."""
    L = make_layout(layout)
    d = dims(L)
    qkv = (d["B"], d["H"], d["Sp"], d["D"])
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, torch.bfloat16, qkv)
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(d["D"])
    if out is None:
        out = torch.empty(qkv, dtype=torch.bfloat16, device=q.device)
    if lse is None and with_lse:
        lse = torch.empty((d["B"], d["H"], d["Sp"]), dtype=torch.float32, device=q.device)
    workspace = _attn_workspace(L, q.device, workspace)
    rc = load().bsa_dense_fwd(ctypes.byref(L), _ptr(q), _ptr(k), _ptr(v), float(softmax_scale),
                              _ptr(out), _ptr(lse), _ptr(err_flag), _ptr(workspace),
                              _stream(stream))
    _check("bsa_dense_fwd", rc)
    return out, lse


def sparse_attention(layout, q, k, v, top_p, flags, eps=1e-8, softmax_scale=None, stream=None):
    """The whole path: scores -> mask -> block-sparse attention.  Returns a dict."""
    qc, kc, probs = block_scores(layout, q, k, stream=stream)
    sel = build_mask(layout, probs, top_p, flags, eps, stream=stream)
    out, lse = attention_fwd(layout, q, k, v, sel["kv_index"], sel["kv_count"], softmax_scale,
                             stream=stream)
    sel.update(q_centroids=qc, k_centroids=kc, probs=probs, out=out, lse=lse)
    return sel


def pipeline_workspace_bytes(layout, heads_per_group):
    return int(load().bsa_pipeline_workspace_bytes(ctypes.byref(make_layout(layout)),
                                                   int(heads_per_group)))


def _need_host(t, name, dtype, shape):
    if t.dtype != dtype:
        raise TypeError("%s: expected %s, got %s" % (name, dtype, t.dtype))
    if t.is_cuda:
        raise ValueError("%s must be a host tensor" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if tuple(t.shape) != tuple(shape):
        raise ValueError("%s: expected shape %s, got %s" % (name, tuple(shape), tuple(t.shape)))


def sparse_attention_host(layout, q, k, v, top_p, flags, eps=1e-8, softmax_scale=None,
                          heads_per_group=2, out=None, entropy=None, entropy_norm=None,
                          kv_count=None, err_flag=None, workspace=None, stream=None,
                          h2d_stream=None, d2h_stream=None, device=None):
    """bsa_sparse_attention_host: the whole path on HOST q, k, v (page-locked
    for overlap), writing HOST out (and optional entropy / kv_count).  Queued
    on `stream` (default: the current stream of `device`); returns a dict of
    the host outputs, valid once that stream is synchronised."""
    L = make_layout(layout)
    B, H, Sp, D = L.batch, L.heads, L.seq_pad, L.head_dim
    Cq = Sp // L.q_block
    for n, t in (("q", q), ("k", k), ("v", v)):
        _need_host(t, n, torch.bfloat16, (B, H, Sp, D))
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    if out is None:
        out = torch.empty((B, H, Sp, D), dtype=torch.bfloat16, pin_memory=True)
    _need_host(out, "out", torch.bfloat16, (B, H, Sp, D))
    if entropy is not None:
        _need_host(entropy, "entropy", torch.float32, (B, H))
    if entropy_norm is not None:
        _need_host(entropy_norm, "entropy_norm", torch.float32, (B, H))
    if kv_count is not None:
        _need_host(kv_count, "kv_count", torch.int32, (B, H, Cq))
    if err_flag is not None:
        _need_host(err_flag, "err_flag", torch.int32, (1,))
    nbytes = pipeline_workspace_bytes(L, heads_per_group)
    if nbytes == 0:
        raise BsaError("bsa_pipeline_workspace_bytes", BSA_ERR_INVALID_ARG)
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    elif workspace.numel() * workspace.element_size() < nbytes:
        raise ValueError("workspace: %d bytes needed" % nbytes)
    scale = 1.0 / math.sqrt(D) if softmax_scale is None else float(softmax_scale)
    if len(top_p) != H:
        raise ValueError("top_p: expected %d values" % H)
    tp = (ctypes.c_float * H)(*[float(x) for x in top_p])
    cs = torch.cuda.current_stream(dev) if stream is None else stream
    hs = cs if h2d_stream is None else h2d_stream
    ds = cs if d2h_stream is None else d2h_stream
    rc = load().bsa_sparse_attention_host(
        ctypes.byref(L), int(heads_per_group), _ptr(q), _ptr(k), _ptr(v),
        ctypes.cast(tp, ctypes.c_void_p), int(flags), float(eps), scale, _ptr(out), _ptr(entropy),
        _ptr(entropy_norm), _ptr(kv_count), _ptr(err_flag), _ptr(workspace), nbytes,
        ctypes.c_void_p(cs.cuda_stream), ctypes.c_void_p(hs.cuda_stream),
        ctypes.c_void_p(ds.cuda_stream))
    _check("bsa_sparse_attention_host", rc)
    return dict(out=out, entropy=entropy, entropy_norm=entropy_norm, kv_count=kv_count,
                err_flag=err_flag, workspace=workspace)
