"""The C ABI on a host without a GPU: the library loads, exports every symbol
include/bsa.h declares, and rejects bad arguments before launching anything."""
import ctypes

import pytest

from block_sparse_attention_45_b200 import binding as bsa
from block_sparse_attention_45_b200 import synth


def test_library_exports_every_declared_symbol():
    lib = bsa.load()
    names = bsa.declared_symbols()
    assert {"bsa_block_scores", "bsa_build_mask", "bsa_attention_fwd", "bsa_dense_fwd"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n
    assert lib.bsa_version() >= 100
    for s in range(5):
        assert bsa.status_string(s).startswith("BSA_")


def _layout(**kw):
    d = synth.WORKLOADS["tiny"].layout()
    d.update(kw)
    return bsa.make_layout(d)


FAKE = ctypes.c_void_p(0x10000)      # never dereferenced: validation fails first
MISALIGNED = ctypes.c_void_p(0x10002)


@pytest.mark.parametrize("kw,expect", [
    (dict(head_dim=96), bsa.BSA_ERR_UNSUPPORTED),
    (dict(q_block=32), bsa.BSA_ERR_UNSUPPORTED),
    (dict(heads=0), bsa.BSA_ERR_INVALID_ARG),
    (dict(heads=257), bsa.BSA_ERR_UNSUPPORTED),
    (dict(seq_pad=300), bsa.BSA_ERR_INVALID_ARG),          # not a multiple of the block
    (dict(seq_len=200), bsa.BSA_ERR_INVALID_ARG),          # a whole empty block at the end
    (dict(seq_len=400), bsa.BSA_ERR_INVALID_ARG),          # seq_pad < seq_len
    (dict(text_len=300), bsa.BSA_ERR_INVALID_ARG),         # text + frames beyond seq_len
    (dict(num_frames=-1), bsa.BSA_ERR_INVALID_ARG),
])
def test_bad_layouts_are_rejected(kw, expect):
    L = _layout(**kw)
    lib = bsa.load()
    assert lib.bsa_dense_fwd(ctypes.byref(L), FAKE, FAKE, FAKE, 0.125, FAKE, None, None, None, None) == expect
    assert lib.bsa_block_scores(ctypes.byref(L), FAKE, FAKE, FAKE, FAKE, FAKE, None) == expect
    assert lib.bsa_build_mask_workspace_bytes(ctypes.byref(L)) == 0


def test_bad_pointers_are_rejected():
    L = _layout()
    lib = bsa.load()
    r = ctypes.byref(L)
    assert lib.bsa_dense_fwd(r, MISALIGNED, FAKE, FAKE, 0.125, FAKE, None, None, None, None) == bsa.BSA_ERR_INVALID_ARG
    assert lib.bsa_dense_fwd(r, None, FAKE, FAKE, 0.125, FAKE, None, None, None, None) == bsa.BSA_ERR_INVALID_ARG
    assert lib.bsa_dense_fwd(r, FAKE, FAKE, FAKE, -1.0, FAKE, None, None, None, None) == bsa.BSA_ERR_INVALID_ARG
    assert lib.bsa_attention_fwd(r, FAKE, FAKE, FAKE, None, FAKE, 0.125, FAKE, None, None,
                                 None, None) == bsa.BSA_ERR_INVALID_ARG
    assert lib.bsa_dense_fwd(r, FAKE, FAKE, FAKE, 0.125, FAKE, None, None, MISALIGNED,
                             None) == bsa.BSA_ERR_INVALID_ARG
    assert lib.bsa_block_scores(r, FAKE, FAKE, FAKE, FAKE, MISALIGNED, None) == bsa.BSA_ERR_INVALID_ARG
    tp = (ctypes.c_float * 2)(0.5, 0.5)
    tpv = ctypes.cast(tp, ctypes.c_void_p)
    # entropy requested without a workspace; unknown flag bit; no top_p
    assert lib.bsa_build_mask(r, FAKE, tpv, 3, 1e-8, None, FAKE, FAKE, FAKE, None, None,
                              None) == bsa.BSA_ERR_INVALID_ARG
    assert lib.bsa_build_mask(r, FAKE, tpv, 8, 1e-8, None, FAKE, FAKE, None, None, None,
                              None) == bsa.BSA_ERR_INVALID_ARG
    assert lib.bsa_build_mask(r, FAKE, None, 3, 1e-8, None, FAKE, FAKE, None, None, None,
                              None) == bsa.BSA_ERR_INVALID_ARG
    nan_tp = (ctypes.c_float * 2)(float("nan"), 0.5)
    assert lib.bsa_build_mask(r, FAKE, ctypes.cast(nan_tp, ctypes.c_void_p), 3, 1e-8, None, FAKE,
                              FAKE, None, None, None, None) == bsa.BSA_ERR_INVALID_ARG


def test_workspace_size():
    L = _layout()
    assert bsa.load().bsa_attention_workspace_bytes(ctypes.byref(L)) == 256
    # one fp32 per (b, h, query block), rounded up to 256 bytes
    assert bsa.load().bsa_build_mask_workspace_bytes(ctypes.byref(L)) == 256
    w = synth.WORKLOADS["hunyuan"]
    L = bsa.make_layout(w)
    assert bsa.load().bsa_build_mask_workspace_bytes(ctypes.byref(L)) == -(-24 * 931 * 4 // 256) * 256


def _host_call(lib, L, hpg=1, q=FAKE, out=FAKE, top_p=None, flags=3, eps=1e-8, scale=0.125,
               ws=ctypes.c_void_p(0x100000), ws_bytes=1 << 40):
    tp = (ctypes.c_float * L.heads)(*([0.5] * L.heads)) if top_p is None else top_p
    return lib.bsa_sparse_attention_host(
        ctypes.byref(L), hpg, q, FAKE, FAKE, ctypes.cast(tp, ctypes.c_void_p), flags, eps, scale,
        out, None, None, None, None, ws, ws_bytes, None, None, None)


def test_pipeline_entry_point_validates_before_any_cuda_call():
    lib = bsa.load()
    L = _layout()
    # every rejection below happens on the host, before a stream or event is touched
    assert _host_call(lib, _layout(head_dim=96)) == bsa.BSA_ERR_UNSUPPORTED
    assert _host_call(lib, _layout(seq_len=200)) == bsa.BSA_ERR_INVALID_ARG
    assert _host_call(lib, L, hpg=0) == bsa.BSA_ERR_INVALID_ARG
    assert _host_call(lib, L, q=None) == bsa.BSA_ERR_INVALID_ARG
    assert _host_call(lib, L, out=None) == bsa.BSA_ERR_INVALID_ARG
    assert _host_call(lib, L, ws=None) == bsa.BSA_ERR_INVALID_ARG
    assert _host_call(lib, L, ws=ctypes.c_void_p(0x100010)) == bsa.BSA_ERR_INVALID_ARG  # not 256-aligned
    need = lib.bsa_pipeline_workspace_bytes(ctypes.byref(L), 1)
    assert _host_call(lib, L, ws_bytes=need - 1) == bsa.BSA_ERR_INVALID_ARG
    assert _host_call(lib, L, flags=8) == bsa.BSA_ERR_INVALID_ARG
    assert _host_call(lib, L, eps=-1.0) == bsa.BSA_ERR_INVALID_ARG
    assert _host_call(lib, L, scale=0.0) == bsa.BSA_ERR_INVALID_ARG
    nan_tp = (ctypes.c_float * 2)(0.5, float("nan"))
    assert _host_call(lib, L, top_p=nan_tp) == bsa.BSA_ERR_INVALID_ARG


def test_pipeline_workspace_size():
    lib = bsa.load()
    w = synth.WORKLOADS["hunyuan"]
    L = bsa.make_layout(w)
    assert lib.bsa_pipeline_workspace_bytes(ctypes.byref(L), 0) == 0
    assert lib.bsa_pipeline_workspace_bytes(ctypes.byref(_layout(head_dim=96)), 1) == 0
    one = lib.bsa_pipeline_workspace_bytes(ctypes.byref(L), 1)
    two = lib.bsa_pipeline_workspace_bytes(ctypes.byref(L), 2)
    # two slots, each holding q, k, v, out of the group plus its selection buffers
    per_head = 4 * w.seq_pad * w.head_dim * 2
    assert one > 2 * per_head and two > 2 * (2 * per_head)
    assert two - one >= 2 * per_head
    # a group larger than H is clamped to H
    assert lib.bsa_pipeline_workspace_bytes(ctypes.byref(L), 1000) == \
        lib.bsa_pipeline_workspace_bytes(ctypes.byref(L), w.heads)


def test_eg_entry_points_validate_before_any_cuda_call():
    lib = bsa.load()
    L = _layout()
    r = ctypes.byref(L)
    tp = (ctypes.c_float * 2)(0.5, 0.5)
    tpv = ctypes.cast(tp, ctypes.c_void_p)
    ws = ctypes.c_void_p(0x100000)

    def eg(probs=FAKE, vnorm=None, top=tpv, pool_p=0.9, flags=3, idx=FAKE, cnt=FAKE, w=ws):
        return lib.bsa_build_mask_eg(r, probs, vnorm, top, pool_p, flags, 1e-8, None, idx, cnt,
                                     None, None, None, w, None)
    assert eg(probs=None) == bsa.BSA_ERR_INVALID_ARG
    assert eg(top=None) == bsa.BSA_ERR_INVALID_ARG
    assert eg(idx=None) == bsa.BSA_ERR_INVALID_ARG
    assert eg(w=None) == bsa.BSA_ERR_INVALID_ARG
    assert eg(w=ctypes.c_void_p(0x100010)) == bsa.BSA_ERR_INVALID_ARG     # not 256-aligned
    assert eg(vnorm=MISALIGNED) == bsa.BSA_ERR_INVALID_ARG
    assert eg(flags=8) == bsa.BSA_ERR_INVALID_ARG
    assert eg(pool_p=float("nan")) == bsa.BSA_ERR_INVALID_ARG
    nan_tp = (ctypes.c_float * 2)(float("nan"), 0.5)
    assert eg(top=ctypes.cast(nan_tp, ctypes.c_void_p)) == bsa.BSA_ERR_INVALID_ARG
    bad = _layout(head_dim=96)
    assert lib.bsa_build_mask_eg(ctypes.byref(bad), FAKE, None, tpv, 0.9, 3, 1e-8, None, FAKE, FAKE,
                                 None, None, None, ws, None) == bsa.BSA_ERR_UNSUPPORTED
    assert lib.bsa_value_norms(r, None, FAKE, None) == bsa.BSA_ERR_INVALID_ARG
    assert lib.bsa_value_norms(r, MISALIGNED, FAKE, None) == bsa.BSA_ERR_INVALID_ARG
    assert lib.bsa_value_norms(ctypes.byref(bad), FAKE, FAKE, None) == bsa.BSA_ERR_UNSUPPORTED
    # workspace: per-row tie counts + a 256-bin level-1 histogram per head + one pool state and
    # 4096-bin histogram per batch entry
    assert lib.bsa_build_mask_eg_workspace_bytes(ctypes.byref(bad)) == 0
    w = synth.WORKLOADS["hunyuan"]
    n = lib.bsa_build_mask_eg_workspace_bytes(ctypes.byref(bsa.make_layout(w)))
    rows = w.heads * (w.seq_pad // w.q_block)
    assert n >= rows * 4 + w.heads * 256 * 16 + 4096 * 16 and n % 256 == 0
    # the domain entry: the same checks, plus the domain; the EG domain's workspace is EG's,
    # per-head pools need one 4096-bin histogram per head
    assert lib.bsa_build_mask_domain_workspace_bytes(ctypes.byref(bsa.make_layout(w)), bsa.DOMAIN_EG) == n
    assert lib.bsa_build_mask_domain_workspace_bytes(ctypes.byref(bsa.make_layout(w)), 5) == 0
    assert lib.bsa_build_mask_domain_workspace_bytes(ctypes.byref(bsa.make_layout(w)), -1) == 0
    assert lib.bsa_build_mask_domain_workspace_bytes(ctypes.byref(bad), bsa.DOMAIN_ALL) == 0
    nh = lib.bsa_build_mask_domain_workspace_bytes(ctypes.byref(bsa.make_layout(w)), bsa.DOMAIN_HEAD)
    assert nh >= n + (w.heads - 1) * 4096 * 16

    def dom(domain=bsa.DOMAIN_GROUPED, probs=FAKE, top=tpv, idx=FAKE, w=ws):
        return lib.bsa_build_mask_domain(r, domain, probs, None, top, 0.9, 3, 1e-8, None, idx, FAKE,
                                         None, None, None, w, None)
    for d in (-1, 5, 100):
        assert dom(domain=d) == bsa.BSA_ERR_INVALID_ARG
    assert dom(probs=None) == bsa.BSA_ERR_INVALID_ARG
    assert dom(top=None) == bsa.BSA_ERR_INVALID_ARG
    assert dom(idx=None) == bsa.BSA_ERR_INVALID_ARG
    assert dom(w=ctypes.c_void_p(0x100010)) == bsa.BSA_ERR_INVALID_ARG


def test_clustered_scores_validate_before_any_cuda_call():
    lib = bsa.load()
    L = _layout()
    r = ctypes.byref(L)
    ws = ctypes.c_void_p(0x100000)

    def cl(q=FAKE, nsub=4, iters=3, cent=FAKE, size=FAKE, kc=FAKE, probs=FAKE, w=ws):
        return lib.bsa_block_scores_clustered(r, q, FAKE, nsub, iters, cent, size, kc, probs, w, None)
    assert cl(q=None) == bsa.BSA_ERR_INVALID_ARG
    assert cl(cent=None) == bsa.BSA_ERR_INVALID_ARG
    assert cl(size=None) == bsa.BSA_ERR_INVALID_ARG
    assert cl(w=None) == bsa.BSA_ERR_INVALID_ARG
    assert cl(w=ctypes.c_void_p(0x100010)) == bsa.BSA_ERR_INVALID_ARG
    assert cl(cent=MISALIGNED) == bsa.BSA_ERR_INVALID_ARG
    assert cl(iters=0) == bsa.BSA_ERR_INVALID_ARG
    assert cl(nsub=3) == bsa.BSA_ERR_UNSUPPORTED
    assert cl(nsub=32) == bsa.BSA_ERR_UNSUPPORTED
    assert cl(nsub=0) == bsa.BSA_ERR_UNSUPPORTED
    assert lib.bsa_block_scores_clustered_workspace_bytes(r, 3) == 0
    w = synth.WORKLOADS["tiny"]
    cq, ck = w.seq_pad // w.q_block, w.seq_pad // w.k_block
    assert lib.bsa_block_scores_clustered_workspace_bytes(r, 4) >= \
        w.batch * w.heads * cq * 4 * ck * 4


def test_frame_scores_validate_before_any_cuda_call():
    lib = bsa.load()
    win = synth.WINDOWS["selfforcing"]
    L = bsa.make_layout(win)
    r = ctypes.byref(L)
    ws = ctypes.c_void_p(0x100000)

    def fs(lay=r, q=FAKE, alpha=FAKE, w=ws, scale=0.088, stride=1):
        return lib.bsa_frame_scores(lay, q, FAKE, scale, stride, alpha, w, None)
    assert fs(q=None) == bsa.BSA_ERR_INVALID_ARG
    assert fs(alpha=None) == bsa.BSA_ERR_INVALID_ARG
    assert fs(w=None) == bsa.BSA_ERR_INVALID_ARG
    assert fs(w=ctypes.c_void_p(0x100010)) == bsa.BSA_ERR_INVALID_ARG
    assert fs(stride=0) == bsa.BSA_ERR_INVALID_ARG
    assert fs(scale=float("inf")) == bsa.BSA_ERR_INVALID_ARG
    # not a key window: text tokens, one frame, or tokens outside the frames
    for kw in (dict(text_len=64, seq_len=win.seq_len + 64, seq_pad=win.seq_pad + 128),
               dict(num_frames=1, seq_len=win.tokens_per_frame, seq_pad=1664),
               dict(seq_len=win.seq_len - 8, num_frames=4, seq_pad=win.seq_pad)):
        d = win.layout()
        d.update(kw)
        assert fs(lay=ctypes.byref(bsa.make_layout(d))) == bsa.BSA_ERR_INVALID_ARG, kw
    n = lib.bsa_frame_scores_workspace_bytes(r)
    assert n >= 2 * 2 * win.heads * win.seq_pad * win.head_dim and n % 256 == 0


def test_sampling_entry_points_validate_before_any_cuda_call():
    lib = bsa.load()
    L = _layout()
    r = ctypes.byref(L)

    def smp(probs=FAKE, budget=4.0, flags=3, idx=FAKE, wt=FAKE, cnt=FAKE):
        return lib.bsa_build_mask_sampled(r, probs, budget, 7, flags, None, idx, wt, cnt, None)
    assert smp(probs=None) == bsa.BSA_ERR_INVALID_ARG
    assert smp(idx=None) == bsa.BSA_ERR_INVALID_ARG
    assert smp(wt=None) == bsa.BSA_ERR_INVALID_ARG
    assert smp(cnt=None) == bsa.BSA_ERR_INVALID_ARG
    assert smp(wt=MISALIGNED) == bsa.BSA_ERR_INVALID_ARG
    assert smp(flags=8) == bsa.BSA_ERR_INVALID_ARG
    assert smp(budget=-1.0) == bsa.BSA_ERR_INVALID_ARG
    assert smp(budget=float("nan")) == bsa.BSA_ERR_INVALID_ARG
    assert smp(budget=float("inf")) == bsa.BSA_ERR_INVALID_ARG
    bad = _layout(head_dim=96)
    assert lib.bsa_build_mask_sampled(ctypes.byref(bad), FAKE, 4.0, 7, 0, None, FAKE, FAKE, FAKE,
                                      None) == bsa.BSA_ERR_UNSUPPORTED

    def wat(q=FAKE, idx=FAKE, wt=FAKE, cnt=FAKE, scale=0.125, out=FAKE):
        return lib.bsa_attention_fwd_weighted(r, q, FAKE, FAKE, idx, wt, cnt, scale, out, None, None,
                                              None, None)
    assert wat(q=None) == bsa.BSA_ERR_INVALID_ARG
    assert wat(wt=None) == bsa.BSA_ERR_INVALID_ARG
    assert wat(idx=None) == bsa.BSA_ERR_INVALID_ARG
    assert wat(wt=MISALIGNED) == bsa.BSA_ERR_INVALID_ARG
    assert wat(scale=0.0) == bsa.BSA_ERR_INVALID_ARG
    assert wat(out=MISALIGNED) == bsa.BSA_ERR_INVALID_ARG


def test_calls_fail_loudly_without_the_library(monkeypatch):
    monkeypatch.setattr(bsa, "_LIB", None)
    monkeypatch.setattr(bsa, "LIB_PATH", "/nonexistent/libbsa.so")
    with pytest.raises(RuntimeError, match="not built"):
        bsa.load()


def test_binding_types_every_declared_entry_point():
    """Every function of include/bsa.h gets argtypes and restype in the binding,
    so no pointer or size crosses the boundary as a default C int."""
    lib = bsa.load()
    for name in sorted(bsa.declared_symbols()):
        fn = getattr(lib, name)
        assert fn.argtypes is not None, name
        assert fn.restype is not None, name
