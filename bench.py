"""Benchmark of the dynamic block-sparse attention path on B200.

One step = one pass of the whole path over one batch: bsa_block_scores
(centroids + P'), bsa_build_mask (top-p, text keep, frame-0 override, entropy,
lists) and bsa_attention_fwd (exact attention over the selected blocks), on
seeded synthetic inputs already resident in HBM.  Default workload: the
HunyuanVideo-shaped sequence (B=1, H=24, D=128, 119,056 tokens, per-head top-p
calibrated to 90 % skipped key blocks).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--no-e2e] [--no-cpu-baseline]

Prints ONE JSON line on rank 0.  `value` is the computed attention TFLOP/s of
the whole step (selected block pairs x 4*bq*bk*D FLOP / step time) summed over
ranks; `ms_per_step` is the step time (max over ranks).  With torchrun
(N > 1) the default `--shard heads` splits the heads of the one problem over
the ranks (the path is independent per head, so no collective touches the data;
strong scaling); `--shard replicas` runs an independent copy per rank (weak
scaling).  `--impl reference` times the CPU oracle on a bounded sample of the
same workload (rank 0 only).
"""
import argparse
import dataclasses
import glob
import json
import re
import os
import signal
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "block-sparse attn ms/call and computed TFLOP/s (% of B200 BF16 peak) at ~90% sparsity"
UNIT = "TFLOP/s"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="hunyuan")
    ap.add_argument("--heads", type=int, default=None,
                    help="run only heads 0 .. N-1 of the workload (a reduced case, e.g. for ncu)")
    ap.add_argument("--shard", default="heads", choices=["heads", "replicas"],
                    help="N > 1: split the heads of the one problem across the ranks (heads), "
                         "or run one whole copy per rank (replicas)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-group", type=int, default=1,
                    help="heads per group of the pipelined host-buffer call timed as e2e")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--no-profile", action="store_true",
                    help="skip the head-profiling context measurement")
    ap.add_argument("--no-domains", action="store_true",
                    help="skip the competition-domain context measurement")
    ap.add_argument("--selection", default="top_p", choices=["top_p", "eg", "sampled"],
                    help="per-row top-p (bsa_build_mask), entropy-guided grouped selection "
                         "(bsa_value_norms + bsa_build_mask_eg), or importance sampling with "
                         "inverse-probability weights (bsa_build_mask_sampled + "
                         "bsa_attention_fwd_weighted) inside the step")
    ap.add_argument("--subclusters", type=int, default=1,
                    help="query sub-clusters per block for the block scores (1: block centroids, "
                         "bsa_block_scores; 2-16: bsa_block_scores_clustered)")
    ap.add_argument("--kmeans-iters", type=int, default=3)
    ap.add_argument("--budget", type=float, default=None,
                    help="per-row budget K of the sampler (default: calibrated so the expected "
                         "density matches the per-row top-p selection)")
    ap.add_argument("--pool-p", type=float, default=None,
                    help="threshold of the low-entropy pool (default: the mean per-head top-p)")
    return ap.parse_args()


def load_top_p(w):
    if w.top_p is not None:
        return [float(w.top_p)] * w.heads
    cal = json.load(open(os.path.join(ROOT, "tests", "golden", "top_p_calibrated.json")))
    return [float(x) for x in cal[w.name]["top_p"]]


def measured_peaks():
    try:
        return json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
    except OSError:
        return None


def flops_per_pair(w):
    return 4.0 * w.q_block * w.k_block * w.head_dim


def max_over_ranks(value, device=None):
    """The job's time is the slowest rank's (torch.distributed MAX all-reduce)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tflops(flops_per_rank_step, world, ms_per_step):
    """Whole-job throughput: every rank runs its own problem (weak scaling)."""
    return world * flops_per_rank_step / (ms_per_step * 1e-3) / 1e12


def sum_over_ranks(value, device=None):
    """Sum of a per-rank count over the job (torch.distributed SUM all-reduce)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def head_shard(heads, world, rank):
    """Heads [h0, h1) of rank `rank` when the heads of one problem are split over
    `world` ranks: contiguous, sizes differing by at most one.  The path is
    independent per (batch, head), so the shards need no exchange."""
    return rank * heads // world, (rank + 1) * heads // world


# ---------------------------------------------------------------- CPU oracle legs

def oracle_sample(w, x, top_p, budget_s=20.0):
    """Time the oracle (as it stands) on a bounded sample of the workload.

    Selection for one head (pool, P', entropy, top-p, overrides, lists) plus
    sparse attention for query blocks of that head, taken in a seeded random
    order until about budget_s of attention work is done.  Returns computed
    attention TFLOP/s over the sampled blocks, the sample description and the
    thread count.
    """
    import oracle
    ora = oracle.default()
    L1 = dict(w.layout(), heads=1, batch=1)
    q1, k1, v1 = x["q"][:1, :1], x["k"][:1, :1], x["v"][:1, :1]
    t0 = time.perf_counter()
    sel = ora.select(L1, q1, k1, top_p[:1], w.flags)
    t_sel = time.perf_counter() - t0
    cq = w.seq_pad // w.q_block
    order = np.random.default_rng(0).permutation(cq)
    chunk = max(1, ora.num_threads())     # the oracle spreads query blocks over its threads
    done, pairs, t_attn = [], 0, 0.0
    for c0 in range(0, cq, chunk):
        rows = order[c0:c0 + chunk].astype(np.int64)
        t1 = time.perf_counter()
        ora.attention(L1, q1, k1, v1, sel["mask"], rows=rows)
        t_attn += time.perf_counter() - t1
        done.extend(int(i) for i in rows)
        pairs += int(sel["kv_count"][0, 0, rows].sum())
        if t_attn >= budget_s:
            break
    fl = pairs * flops_per_pair(w)
    # the sampled blocks' share of one head's selection time is charged pro rata
    t_total = t_attn + t_sel * len(done) / cq
    return dict(tflops=fl / t_total / 1e12, seconds=t_total, blocks=len(done), pairs=pairs,
                threads=ora.num_threads(), t_select_head=t_sel)


def reference_arm(args, w):
    """--impl reference: the CPU oracle as the reference arm (rank 0 only)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from block_sparse_attention_45_b200 import synth
    top_p = load_top_p(w)
    x = synth.generate(w, heads=[0])
    per = max(2.0, 60.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        oracle_sample(w, x, top_p, budget_s=per)
    vals, secs, desc = [], 0.0, None
    for _ in range(args.steps):
        r = oracle_sample(w, x, top_p, budget_s=per)
        vals.append(r["tflops"])
        secs += r["seconds"]
        desc = r
    v = float(np.mean(vals))
    sample = ("oracle on head 0 of %s: selection for the head + exact sparse attention for %d "
              "random query blocks (%d selected block pairs) per step" % (w.name, desc["blocks"],
                                                                          desc["pairs"]))
    line = dict(metric=METRIC, value=v, unit=UNIT, n_gpus=args.gpus, steps=args.steps,
                warmup=args.warmup, ms_per_step=secs / args.steps * 1e3, higher_is_better=True,
                scaling="weak", vs_baseline=None, dtype="f64", data="synthetic", impl="reference",
                config=dict(workload=w.name, **{k: v for k, v in w.layout().items()}),
                cpu_baseline=dict(value=v, unit=UNIT, cores=desc["threads"], kind="oracle",
                                  sample=sample),
                e2e=dict(value=v, unit=UNIT, h2d_bytes_per_step=0, d2h_bytes_per_step=0))
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def wait_first_sample(self, timeout=5.0):
        """Block until nvidia-smi has written its first sample (its start-up takes a
        while), so that a short timed region still falls between samples."""
        if self.proc is None:
            return
        t0 = time.time()
        while time.time() - t0 < timeout and self.proc.poll() is None:
            try:
                if os.path.getsize(self.path) > 0:
                    return
            except OSError:
                return
            time.sleep(0.02)

    def stop(self):
        if self.proc is None:
            return None
        self.proc.send_signal(signal.SIGTERM)
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            f = [s.strip() for s in line.split(",")]
            if len(f) < 9:
                continue
            try:
                rows.append((float(f[1]), float(f[2]), f[5:9]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i in range(4) if r[i] == "Active"})
        sm = [r[0] for r in rows]
        return dict(sm_mhz=float(np.median(sm)), sm_max_mhz=max(r[1] for r in rows),
                    samples=len(rows), reasons=reasons)


# ---------------------------------------------------------------- our arm

def our_arm(args, w):
    import torch
    import torch.distributed as dist
    from block_sparse_attention_45_b200 import binding as bsa
    from block_sparse_attention_45_b200 import synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)

    top_p = load_top_p(w)
    if args.heads:   # a reduced case: the first heads of the workload, their own p and seeds
        w = dataclasses.replace(w, heads=min(args.heads, w.heads))
        top_p = list(top_p[:w.heads])
    w_job = w
    split = world > 1 and args.shard == "heads"
    h0, h1 = head_shard(w.heads, world, rank) if split else (0, w.heads)
    if split:   # this rank's heads of the one problem (each head keeps its own seeds)
        w = dataclasses.replace(w, heads=h1 - h0)
        top_p = list(top_p[h0:h1])
    x = synth.generate(w, heads=range(h0, h1))
    host = {k: torch.from_numpy(v.view(np.int16)).view(torch.bfloat16) for k, v in x.items()}
    q, k, v = (host[n].to(dev) for n in ("q", "k", "v"))
    B, H, Sp, D = w.batch, w.heads, w.seq_pad, w.head_dim
    Cq, Ck = Sp // w.q_block, Sp // w.k_block
    f32 = dict(dtype=torch.float32, device=dev)
    qc = torch.empty((B, H, Cq, D), **f32)
    kc = torch.empty((B, H, Ck, D), **f32)
    probs = torch.empty((B, H, Cq, Ck), **f32)
    mask = torch.empty((B, H, Cq, Ck), dtype=torch.uint8, device=dev)
    kv_index = torch.empty((B, H, Cq, Ck), dtype=torch.int32, device=dev)
    kv_count = torch.empty((B, H, Cq), dtype=torch.int32, device=dev)
    ent = torch.empty((B, H), **f32)
    ent_n = torch.empty((B, H), **f32)
    ws = torch.empty(bsa.workspace_bytes(w), dtype=torch.uint8, device=dev)
    eg = args.selection == "eg"
    pool_p = float(np.mean(top_p)) if args.pool_p is None else args.pool_p
    vnorm = torch.empty((B, H, Ck), **f32)
    low = torch.empty((B, H), dtype=torch.uint8, device=dev)
    ws_eg = torch.empty(bsa.eg_workspace_bytes(w), dtype=torch.uint8, device=dev)

    sampled = args.selection == "sampled"
    kv_weight = torch.empty((B, H, Cq, Ck), **f32)
    budget = args.budget

    def select_eg():
        bsa.value_norms(w, v, vnorm, stream=stream)
        bsa.build_mask_eg(w, probs, vnorm, top_p, pool_p, w.flags, 1e-8, mask, kv_index, kv_count,
                          ws_eg, stream=stream, entropy=ent, entropy_norm=ent_n, low_heads=low)
    out = torch.empty((B, H, Sp, D), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, H, Sp), **f32)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731

    nsub = args.subclusters
    if nsub > 1:
        sub_c = torch.empty((B, H, Cq, nsub, D), **f32)
        sub_n = torch.empty((B, H, Cq, nsub), dtype=torch.int32, device=dev)
        ws_cl = torch.empty(bsa.clustered_workspace_bytes(w, nsub), dtype=torch.uint8, device=dev)

    def scores(qq, kk):
        if nsub > 1:
            bsa.block_scores_clustered(w, qq, kk, nsub, args.kmeans_iters, sub_c, sub_n, kc, probs,
                                       ws_cl, stream=stream)
        else:
            bsa.block_scores(w, qq, kk, qc, kc, probs, stream=stream)

    def step(qq, kk, vv, marks=None):
        if marks is not None:
            marks[0].record(stream)
        scores(qq, kk)
        if marks is not None:
            marks[1].record(stream)
        if eg:
            select_eg()
        elif sampled:
            step.seed += 1
            bsa.build_mask_sampled(w, probs, budget, step.seed, w.flags, mask, kv_index, kv_weight,
                                   kv_count, stream=stream)
        else:
            bsa.build_mask(w, probs, top_p, w.flags, 1e-8, mask, kv_index, kv_count, ent, ent_n,
                           ws, stream=stream)
        if marks is not None:
            marks[2].record(stream)
        if sampled:
            bsa.attention_fwd_weighted(w, qq, kk, vv, kv_index, kv_weight, kv_count, None, out, lse,
                                       err, stream=stream)
        else:
            bsa.attention_fwd(w, qq, kk, vv, kv_index, kv_count, None, out, lse, err, stream=stream)
        if marks is not None:
            marks[3].record(stream)
    step.seed = 0

    if sampled and budget is None:
        # expected density of the sampler = mean of min(1, K P') (overrides aside), matched to
        # the per-row top-p selection of the same P' by bisection (setup, not timed)
        scores(q, k)
        bsa.build_mask(w, probs, top_p, w.flags, 1e-8, mask, kv_index, kv_count, ent, ent_n, ws,
                       stream=stream)
        target = float(kv_count.sum().item()) / float(B * H * Cq * Ck)
        lo, hi = 0.0, float(Ck)
        for _ in range(50):
            mid = 0.5 * (lo + hi)
            d = float(torch.clamp(probs * mid, max=1.0).mean().item())
            lo, hi = (mid, hi) if d < target else (lo, mid)
        budget = 0.5 * (lo + hi)

    # pool, score, mask, entropy reduce, attention; the entropy-guided selection runs
    # value norms, entropy + level 1, two pool levels, the tie pass and the mask kernel in
    # place of mask + entropy reduce; the sampler one kernel
    launches_per_step = 9 if eg else (4 if sampled else 5)
    if nsub > 1:   # key pooling, k-means, the mixing score kernel in place of pooling + score kernel
        launches_per_step += 1
    for _ in range(max(3, args.warmup)):
        step(q, k, v)
    torch.cuda.synchronize(dev)
    assert int(err.item()) == 0, "device error flag %d" % int(err.item())
    pairs = int(kv_count.sum().item())
    density = pairs / float(B * H * Cq * Ck)
    step_flops = pairs * flops_per_pair(w)

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local])

    marks = [[ev() for _ in range(4)] for _ in range(args.steps)]
    clocks = ClockSampler(local)
    clocks.start()
    clocks.wait_first_sample()
    barrier()
    torch.cuda.synchronize(dev)
    t_start, t_end = ev(), ev()
    t_start.record(stream)
    for s in range(args.steps):
        step(q, k, v, marks[s])
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    time.sleep(0.25)   # one more sample after the timed region
    clk = clocks.stop()
    ms_total = t_start.elapsed_time(t_end)
    # The first timed step starts on an idle GPU right after the synchronize, so its
    # intervals also hold the host's enqueue of the step's first launches; the per-kernel
    # figures (not `value`, which spans every step) use the later steps when there are any.
    first = 1 if args.steps > 1 else 0
    ms_attn = [m[2].elapsed_time(m[3]) for m in marks[first:]]
    ms_scores = [m[0].elapsed_time(m[1]) for m in marks[first:]]
    ms_mask = [m[1].elapsed_time(m[2]) for m in marks[first:]]
    ms_total = max_over_ranks(ms_total, dev)
    ms_step = ms_total / args.steps
    # every rank's selected pairs count toward the job (a head shard's differ from
    # another's); the count is exchanged once, outside the timed region
    job_flops = sum_over_ranks(step_flops, dev)
    job_pairs = int(round(sum_over_ranks(pairs, dev)))
    value = job_flops / (ms_step * 1e-3) / 1e12

    # end to end through the C ABI with HOST buffers: bsa_sparse_attention_host copies
    # Q, K, V in and O (+ entropy) out per head group on two copy streams, overlapped
    # with the kernels of the neighbouring groups
    e2e = None
    if not args.no_e2e and not eg and not sampled:   # the host-buffer call runs per-row top-p
        pin = {n: host[n].pin_memory() for n in ("q", "k", "v")}
        out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        ent_h = torch.empty((B, H), dtype=torch.float32).pin_memory()
        h2d_s, d2h_s = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        nws = bsa.pipeline_workspace_bytes(w, args.e2e_group)
        pws = torch.empty(nws, dtype=torch.uint8, device=dev)

        def e2e_step():
            bsa.sparse_attention_host(w, pin["q"], pin["k"], pin["v"], top_p, w.flags,
                                      heads_per_group=args.e2e_group, out=out_h, entropy=ent_h,
                                      workspace=pws, stream=stream, h2d_stream=h2d_s,
                                      d2h_stream=d2h_s, device=dev)

        e2e_step()
        torch.cuda.synchronize(dev)
        barrier()
        a, b = ev(), ev()
        a.record(stream)
        for _ in range(args.steps):
            e2e_step()
        b.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        ms_e2e = max_over_ranks(a.elapsed_time(b), dev) / args.steps
        h2d = sum_over_ranks(sum(pin[n].numel() * pin[n].element_size() for n in pin), dev)
        d2h = sum_over_ranks(out_h.numel() * out_h.element_size() +
                             ent_h.numel() * ent_h.element_size(), dev)
        e2e = dict(value=job_flops / (ms_e2e * 1e-3) / 1e12, unit=UNIT,
                   ms_per_step=ms_e2e, h2d_bytes_per_step=int(h2d), d2h_bytes_per_step=int(d2h),
                   call="bsa_sparse_attention_host (page-locked host buffers, heads_per_group=%d)"
                        % args.e2e_group)
        del pws

    # the dense path (all key blocks) for context: not part of the step
    dense = None
    if not args.no_dense:
        for _ in range(2):
            bsa.dense_fwd(w, q, k, v, None, out, lse, stream=stream)
        a, b = ev(), ev()
        a.record(stream)
        nd = max(1, min(3, args.steps))
        for _ in range(nd):
            bsa.dense_fwd(w, q, k, v, None, out, lse, stream=stream)
        b.record(stream)
        torch.cuda.synchronize(dev)
        dms = a.elapsed_time(b) / nd
        dflops = B * H * Cq * Ck * flops_per_pair(w)
        dense = dict(ms=dms, tflops=dflops / (dms * 1e-3) / 1e12)

    # the entropy-guided selection for context when it is not the step's selection:
    # value norms + bsa_build_mask_eg on the step's P' (not part of the step)
    eg_ctx = None
    if not eg:
        for _ in range(2):
            select_eg()
        a, b = ev(), ev()
        a.record(stream)
        ne = max(3, args.steps)
        for _ in range(ne):
            select_eg()
        b.record(stream)
        torch.cuda.synchronize(dev)
        eg_pairs = int(kv_count.sum().item())
        eg_ctx = dict(ms=a.elapsed_time(b) / ne, pool_p=pool_p,
                      density=eg_pairs / float(B * H * Cq * Ck),
                      pooled_heads=int(low.sum().item()),
                      call="bsa_value_norms + bsa_build_mask_eg on the step's P'")

    # the pooled selection over each competition domain for context (not part of the step):
    # bsa_build_mask_domain on the step's P' and value norms
    domains_ctx = None
    if not args.no_domains:
        if not eg:
            bsa.value_norms(w, v, vnorm, stream=stream)
        domains_ctx = {}
        pool_of = torch.empty((B, H), dtype=torch.int8, device=dev)
        for dname, dom in (("per_row", bsa.DOMAIN_ROW), ("per_head", bsa.DOMAIN_HEAD),
                           ("grouped", bsa.DOMAIN_GROUPED), ("all_head", bsa.DOMAIN_ALL),
                           ("eg_sparse", bsa.DOMAIN_EG)):
            ws_d = torch.empty(bsa.domain_workspace_bytes(w, dom), dtype=torch.uint8, device=dev)

            def run_domain():
                bsa.build_mask_domain(w, dom, probs, vnorm, top_p, pool_p, w.flags, 1e-8, mask,
                                      kv_index, kv_count, ws_d, stream=stream, entropy=ent,
                                      entropy_norm=ent_n, pool_of=pool_of)
            for _ in range(2):
                run_domain()
            a, b = ev(), ev()
            a.record(stream)
            ne = max(3, args.steps)
            for _ in range(ne):
                run_domain()
            b.record(stream)
            torch.cuda.synchronize(dev)
            domains_ctx[dname] = dict(ms=a.elapsed_time(b) / ne,
                                      density=int(kv_count.sum().item()) / float(B * H * Cq * Ck),
                                      pooled_heads=int((pool_of >= 0).sum().item()))
            del ws_d
        domains_ctx["call"] = "bsa_build_mask_domain on the step's P' and value norms, pool_p %.4g" % pool_p

    # head profiling of autoregressive generation for context (not part of the step): frame
    # attention scores on a Self Forcing-shaped key window (sink + 3 neighbors + current frame),
    # then Dynamic Head Programming on the host
    prof = None
    if not args.no_profile:
        wv = synth.WINDOWS["selfforcing"]
        xv = synth.generate(wv)
        qv, kv = (torch.from_numpy(xv[n].view(np.int16)).view(torch.bfloat16).to(dev)
                  for n in ("q", "k"))
        alpha = torch.empty((wv.batch, wv.heads, 3), dtype=torch.float32, device=dev)
        wsv = torch.empty(bsa.frame_scores_workspace_bytes(wv), dtype=torch.uint8, device=dev)
        for _ in range(3):
            bsa.frame_scores(wv, qv, kv, alpha=alpha, workspace=wsv, stream=stream)
        a, b = ev(), ev()
        a.record(stream)
        npf = 10
        for _ in range(npf):
            bsa.frame_scores(wv, qv, kv, alpha=alpha, workspace=wsv, stream=stream)
        b.record(stream)
        torch.cuda.synchronize(dev)
        pms = a.elapsed_time(b) / npf
        T, F = wv.tokens_per_frame, wv.num_frames
        cq = wv.seq_pad // wv.q_block
        i0, i1 = (F - 1) * T // wv.q_block, (F * T - 1) // wv.q_block
        pflop = wv.batch * wv.heads * (i1 - i0 + 1) * cq * flops_per_pair(wv)
        al = alpha.cpu().numpy()
        labels = bsa.dhp_labels(al[0], wv.heads // 2)
        prof = dict(workload="selfforcing: 12 heads, 5 frames x 1560 tokens, D 128", ms=pms,
                    tflops=pflop / (pms * 1e-3) / 1e12,
                    call="bsa_frame_scores (attention over a one-hot V) + bsa_dhp_labels (host)",
                    dummy_heads=[int(h) for h in np.nonzero(labels == 2)[0]],
                    alpha_mean=[float(v) for v in al.reshape(-1, 3).mean(0)])
        del qv, kv, wsv

    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return

    peaks = measured_peaks()
    job_density = job_pairs / float(B * w_job.heads * Cq * Ck) if split else (
        job_pairs / float(world * B * H * Cq * Ck))
    attn_ms = float(np.mean(ms_attn))
    achieved = step_flops / (attn_ms * 1e-3) / 1e12
    # the attention kernel is timed per call with CUDA events inside a short timed region,
    # so its denominator is the burst GEMM peak; the sustained one and the nominal dense
    # bf16 figure are reported beside it
    if peaks:
        peak, peak_note = peaks["bf16_tflops"], "measured burst (MEASURED_PEAKS.json)"
        sustained = peaks["bf16_tflops_sustained"]
        hbm = peaks["hbm_gbs"]
    else:
        peak, peak_note, sustained, hbm = 1590.0, "fallback burst", 1400.0, 6650.0
    nominal = 2250.0
    traffic = profiled_traffic(w.name)
    # scoring and mask: algorithmic bytes (read Q, K once; write centroids, P'; read P',
    # write mask, lists, counts) over their measured durations
    bytes_scores = 2 * B * H * w.seq_len * D * 2 + 4 * B * H * (Cq + Ck) * D + 4 * B * H * Cq * Ck
    bytes_mask = 4 * B * H * Cq * Ck + B * H * Cq * Ck + 4 * pairs + 4 * B * H * Cq
    if eg:   # value norms read V and write ||c^V||; the pools read them too
        bytes_mask += B * H * w.seq_len * D * 2 + 2 * 4 * B * H * Ck
    line = dict(
        metric=METRIC, value=value, unit=UNIT, n_gpus=world, steps=args.steps, warmup=args.warmup,
        ms_per_step=ms_step, higher_is_better=True, scaling="strong" if split else "weak",
        vs_baseline=None,
        dtype="bf16", data="synthetic (seeded clustered Gaussian Q/K, N(0,1) V; per-head top-p "
                             "calibrated on the CPU oracle)",
        config=dict(workload=w.name, batch=B, heads=w_job.heads, seq_len=w.seq_len, seq_pad=Sp,
                    head_dim=D,
                    q_block=w.q_block, k_block=w.k_block, text_len=w.text_len,
                    frames=w.num_frames, latent=[w.latent_h, w.latent_w],
                    selection=("entropy-guided grouped (pool_p %.4g)" % pool_p) if eg
                              else ("importance-sampled, inverse-probability weights (budget K "
                                    "%.4g per row, a new seed per step)" % budget) if sampled
                              else "per-row top-p",
                    block_scores=("intra-block query clusters: %d per block, %d k-means rounds"
                                  % (nsub, args.kmeans_iters)) if nsub > 1 else "block centroids",
                    density=job_density, skipped=1 - job_density, selected_pairs=job_pairs,
                    computed_tflop_per_step=job_flops / 1e12,
                    dense_equiv_tflop=4.0 * B * w_job.heads * w.seq_len ** 2 * D / 1e12,
                    parallelism=("head-sharded: rank r of %d takes heads [r*%d/%d, (r+1)*%d/%d) of "
                                 "the one problem; no collective on the data path" %
                                 (world, w_job.heads, world, w_job.heads, world)) if split
                                else "replicas, one independent problem per GPU" if world > 1
                                else "1 GPU",
                    l2="inputs (Q, K, V = %.2f GB) larger than the 126 MB L2; no flush" %
                       (3 * B * H * Sp * D * 2 / 1e9)),
        per_kernel_steps=("timed steps 2..%d (step 1 also holds the host's first launches)"
                          % args.steps) if args.steps > 1 else "the one timed step",
        attention=dict(ms=attn_ms, tflops=achieved, dense_equiv_tflops=4.0 * B * H * w.seq_len ** 2
                       * D / (attn_ms * 1e-3) / 1e12, frac_of_burst=achieved / peak,
                       frac_of_sustained=achieved / sustained, frac_of_nominal=achieved / nominal),
        scores=dict(ms=float(np.mean(ms_scores)), gbs=bytes_scores / (np.mean(ms_scores) * 1e-3) / 1e9,
                    frac_hbm=bytes_scores / (np.mean(ms_scores) * 1e-3) / 1e9 / hbm,
                    frac_of_8tbs=bytes_scores / (np.mean(ms_scores) * 1e-3) / 8e12,
                    bytes=bytes_scores),
        mask=dict(ms=float(np.mean(ms_mask)), gbs=bytes_mask / (np.mean(ms_mask) * 1e-3) / 1e9,
                  frac_hbm=bytes_mask / (np.mean(ms_mask) * 1e-3) / 1e9 / hbm,
                  frac_of_8tbs=bytes_mask / (np.mean(ms_mask) * 1e-3) / 8e12, bytes=bytes_mask),
        dense=dense,
        eg_selection=eg_ctx,
        competition_domains=domains_ctx,
        head_profiling=prof,
        roofline=dict(bound="tensor", kernel="attn_kernel", achieved=achieved, peak=peak,
                      unit="TFLOP/s", frac=achieved / peak, peak_source=peak_note,
                      peak_sustained=sustained, frac_of_sustained=achieved / sustained,
                      peak_nominal=nominal, frac_of_nominal=achieved / nominal,
                      traffic=traffic, flop_per_launch=step_flops,
                      flop_per_unit=flops_per_pair(w), units_per_launch=pairs),
        gpu_launches=launches_per_step * args.steps,
        clocks=clk,
        e2e=e2e,
    )
    if not args.no_cpu_baseline and world == 1:
        r = oracle_sample(w, {n: x[n] for n in ("q", "k", "v")}, top_p, budget_s=20.0)
        line["cpu_baseline"] = dict(
            value=r["tflops"], unit=UNIT, cores=r["threads"], kind="oracle",
            sample="oracle on head 0: selection for the head + exact sparse attention for %d random "
                   "query blocks (%d selected block pairs), %.1f s" % (r["blocks"], r["pairs"],
                                                                       r["seconds"]))
    print(json.dumps(line), flush=True)


TRAFFIC_LINE = re.compile(r"traffic: kernel=attn_kernel workload=(\S+) kernel_sha=([0-9a-f]+) "
                          r"bytes_per_launch=(\d+)")


def profiled_traffic(workload):
    """DRAM bytes (read + write) per attention launch from the ncu summaries
    under profiles/, valid only while the kernel source still hashes the same."""
    sha = kernel_sha()
    for f in sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md"))):
        for m in TRAFFIC_LINE.finditer(open(f).read()):
            if m.group(1) == workload and m.group(2) == sha:
                return int(m.group(3))
    return None


def kernel_sha():
    import hashlib
    h = hashlib.sha256()
    for f in ("attention.cu", "ptx.cuh"):
        h.update(open(os.path.join(ROOT, "block_sparse_attention_45_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def main():
    args = parse()
    from block_sparse_attention_45_b200 import synth
    w = synth.WORKLOADS[args.workload]
    if args.impl == "reference":
        reference_arm(args, w)
    else:
        our_arm(args, w)


if __name__ == "__main__":
    main()
