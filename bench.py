"""Benchmark of the INT8-KV segment-causal attention hot path on B200 (one JSON line on stdout).

One step = one pass of the whole path on the production shape (1280x704 -> 880 tokens per latent
frame, 30-frame segment, 16 heads x 128, 18-frame INT8 history, 768-token description head + 8 action
tails of 64):
  a1  nomas_kv_append     quantise-append the finished previous segment (26400 tokens, 18 frames kept)
  a2  nomas_mask_build    dense visibility classes and tile lists
  a4  nomas_attn_prepare  operand pre-pass: current/text K,V to fp16, INT8 history codes widened to fp16
      nomas_attn_run      dense masked attention (steps 1-2 of a segment's denoising)
  a4" nomas_mask_build + nomas_attn_run (NOMAS_MODE_TEXT)   the text query rows of the same joint
      attention (the text stream), over the workspace the video call prepared (same K/V and cache)
  a3  nomas_mask_build    sparse selection (25 % of candidate video blocks)
  a4' nomas_attn_run      block-sparse attention (steps 3-8) over the same prepared workspace: one
      pre-pass serves every call of one cache state and one segment's K/V
(nomas_attn_fwd is exactly prepare + run; they are called separately so each is timed.)
`value` = algorithmic attention FLOPs of the step (visible / selected keys only) / step time, on the
device, inputs resident in HBM.  Inputs (324 MB of bf16 q/k/v per step) exceed the 126 MB L2.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = "C2"
METRIC = "masked attention TFLOP/s (dense + 25% block-sparse step, INT8 KV history) on 1 B200"


def step_config(cfg, world):
    """The `config` object of the JSON line; both arms report the same one."""
    return {"workload": "production_1280x704: 16x128, 30-frame segment (26400 video + 1280 text queries), "
                        "18-frame INT8 history (15840 keys), 768 head + 8 tails x 64; step = append + dense "
                        "mask + dense attention (video rows) + text-row mask + text-row attention + sparse "
                        "selection (25%) + sparse attention",
            "seq_len": cfg.n_query, "heads": cfg.heads, "head_dim": cfg.head_dim,
            "l2": "inputs larger than L2 (324 MB bf16 q/k/v per step)", "parallelism": f"replica x{world}"}
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# Kernel launches of one step: append 1; dense mask 3; prepare 1 (key copy, transposed values and history
# widening in one launch); dense attention 1, plus 1 when the pair kernel splits its partial last wave
# (dense_attention_launches); text mask 3; text attention 2 (the list shares, their merge); sparse mask
# 5; sparse attention 1.
LAUNCHES_PER_STEP = 17


def dense_attention_launches(n_query, heads, sms):
    """Launches of a dense nomas_attn_run at head_dim 128: the library's per-call choice of the pair
    kernel (1.6 x its waves < the block kernel's) and its last-wave split (left-over units run as
    min(16, SMs / left-over, 256 / left-over) >= 2 shares, merged by one more launch)."""
    blocks = (n_query + 127) // 128
    pairs = (blocks + 1) // 2
    wb, wp = -(-blocks * heads // sms), -(-pairs * heads // sms)
    if not 16 * wp < 10 * wb:
        return 1
    units = pairs * heads
    rem = units % sms
    return 2 if units > sms and rem > 0 and min(16, sms // rem, 256 // rem) >= 2 else 1
CSRC = os.path.join(ROOT, "int8_kv_cache_action_b200", "csrc")
COMMON = os.path.join(CSRC, "common.cuh")
TRAFFIC = {  # kernel -> (ncu summary with DRAM bytes per launch, sources whose digest it was taken with)
    "attn": (os.path.join(ROOT, "profiles", "attn_dense_production_traffic.json"),
             (os.path.join(CSRC, "attn_pair.cu"), os.path.join(CSRC, "attn.cuh"), COMMON)),
    "append": (os.path.join(ROOT, "profiles", "append_production_traffic.json"),
               (os.path.join(CSRC, "append.cu"), os.path.join(CSRC, "quant.cuh"), COMMON)),
    "linear": (os.path.join(ROOT, "profiles", "gemm_dit_qkv_traffic.json"),
               (os.path.join(CSRC, "linear.cu"), os.path.join(CSRC, "quant.cuh"), COMMON)),
    "prepare": (os.path.join(ROOT, "profiles", "prepare_production_traffic.json"),
                (os.path.join(CSRC, "prep.cu"), os.path.join(CSRC, "prep.cuh"), COMMON)),
}


def source_digest(paths):
    """Digest of a kernel's sources (its file and the device helpers it includes)."""
    import hashlib
    h = hashlib.sha256()
    for path in paths:
        with open(path, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def measured_traffic(kernel):
    """DRAM bytes per launch of `kernel` from an ncu capture, or None when its sources have changed
    since the counters were taken."""
    path, sources = TRAFFIC[kernel]
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    if d.get("source_sha256_16") != source_digest(sources):
        return None
    return d.get("bytes_per_launch")


def prepare_bytes(cfg, hist_tokens, head_tokens):
    """Algorithmic bytes of nomas_attn_prepare: current and text K, V read as bf16 and written as fp16;
    per history (token, head) the K and V codes read (2 D) with both scales (8 B) and written as fp16
    (4 D) with both scales in age order (8 B); per earlier-head (token, head) the codes read (2 D),
    checked scales (8 B) and fp16 codes written (4 D)."""
    H, D = cfg.heads, cfg.head_dim
    bf = (cfg.n_query + cfg.current.text_len) * H * D * 2 * (2 + 2)
    return bf + hist_tokens * H * (6 * D + 16) + head_tokens * H * (6 * D + 8)


def aggregate_ranks(ms_local, work_per_rank, world, reduce_max=None):
    """Whole-job throughput: the slowest rank's time (max over ranks) and the work of all ranks.
    `reduce_max` maps a local float to its maximum over ranks (identity for one rank)."""
    ms = reduce_max(ms_local) if (reduce_max is not None and world > 1) else ms_local
    return ms, work_per_rank * world / (ms * 1e-3)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def visible_key_sum(cfg, hist_tokens, head_tokens):
    """Sum over query rows of visible keys (dense): closed form per latent frame."""
    T, F = cfg.tokens_per_frame, cfg.current.n_frames
    base = hist_tokens + head_tokens + cfg.n_query + cfg.current.head_len
    tot = 0
    for t in range(F):
        tot += T * (base + sum(a.len for a in cfg.current.tails if a.f0 <= t < a.f1))
    return tot


def text_key_sum(cfg, hist_tokens, head_tokens):
    """Sum over the current text rows of visible keys: a head row sees history, earlier heads, all current
    video and the current head; a row of tail a sees history, earlier heads, the current head, the video
    frames of its window and the tails whose window shares a frame with its own."""
    T, seg = cfg.tokens_per_frame, cfg.current
    ctx = hist_tokens + head_tokens + seg.head_len
    tot = seg.head_len * (ctx + cfg.n_query)
    for a in seg.tails:
        tails = sum(b.len for b in seg.tails if max(a.f0, b.f0) < min(a.f1, b.f1))
        tot += a.len * (ctx + (a.f1 - a.f0) * T + tails)
    return tot


def sparse_key_sum(sel, cfg, hist_tokens, head_tokens):
    """Sum over heads and query rows of kept keys: kept candidate video blocks of the row's query block
    (their valid tokens), every earlier description head, and the row's visible current text."""
    nq, T = cfg.n_query, cfg.tokens_per_frame
    nh = (hist_tokens + 127) // 128
    sel = sel.cpu().numpy()
    H, nqb, keep = sel.shape
    def cand_len(c):
        if c < nh:
            return min(128, hist_tokens - 128 * c)
        c -= nh
        return min(128, nq - 128 * c)
    lens = {}
    tot = 0
    for b in range(nqb):
        rows = range(128 * b, min(128 * b + 128, nq))
        text = sum(cfg.current.head_len + sum(a.len for a in cfg.current.tails if a.f0 <= r // T < a.f1)
                   for r in rows)
        for h in range(H):
            vid = 0
            for c in sel[h, b]:
                c = int(c)
                if c not in lens:
                    lens[c] = cand_len(c)
                vid += lens[c]
            tot += len(rows) * (vid + head_tokens) + text
    return tot


class Clock:
    """Samples nvidia-smi clocks / throttle reasons in the background during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.out = ""
        if self.proc:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out = ""

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in (self.out or "").splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    from int8_kv_cache_action_b200 import _nomas as N
    from int8_kv_cache_action_b200.runtime import KVCache, mask_views, segment_text_of
    from int8_kv_cache_action_b200.workloads import CONFIGS, make_inputs, APPEND_BYTES_PER_TOKEN_HEAD

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    cfg = CONFIGS[WORKLOAD]
    inp = make_inputs(cfg, seed_offset=rank)
    q, kc, vc, kt, vt, qt = (getattr(inp, n).to(dev) for n in ("q", "k_cur", "v_cur", "k_txt", "v_txt", "q_txt"))
    prev = inp.prior[-1]
    pk, pv = prev.k.to(dev), prev.v.to(dev)
    cache = KVCache.for_config(cfg, dev)
    for seg, kv in zip(cfg.prior, inp.prior):
        cache.append(kv.k.to(dev), kv.v.to(dev), seg.n_frames)
    seg = segment_text_of(cfg.current)
    st = torch.cuda.current_stream()
    s = st.cuda_stream
    lay_d = cache.mask_layout(seg, N.NOMAS_MODE_DENSE)
    lay_s = cache.mask_layout(seg, N.NOMAS_MODE_SPARSE, 0.25)
    lay_t = cache.mask_layout(seg, N.NOMAS_MODE_TEXT)
    mbuf_t = torch.empty(lay_t["total_bytes"], dtype=torch.uint8, device=dev)
    mbuf_d = torch.empty(lay_d["total_bytes"], dtype=torch.uint8, device=dev)
    mbuf_s = torch.empty(lay_s["total_bytes"], dtype=torch.uint8, device=dev)
    out_d = torch.empty((cfg.n_query, cfg.heads, cfg.head_dim), dtype=torch.float32, device=dev)
    out_s = torch.empty_like(out_d)
    out_t = torch.empty((cfg.current.text_len, cfg.heads, cfg.head_dim), dtype=torch.float32, device=dev)
    ws = cache.workspace(seg)
    scale = 1.0 / math.sqrt(cfg.head_dim)
    ts, hs = q.stride(0), q.stride(1)
    n_frames_prev = cfg.prior[-1].n_frames

    def check(rc, what):
        if rc != 0:
            raise N.NomasError(rc, what)

    bufs0 = {"q": q, "kc": kc, "vc": vc, "kt": kt, "vt": vt, "qt": qt, "pk": pk, "pv": pv, "out_d": out_d,
             "out_t": out_t, "out_s": out_s}

    def step(ev=None, b=bufs0, stream=None):
        sh = s if stream is None else stream.cuda_stream
        rs = st if stream is None else stream

        def mark(i):
            if ev is not None:
                ev[i].record(rs)

        def prepare():
            check(N.nomas_attn_prepare(cache.handle, seg, b["kc"].data_ptr(), b["vc"].data_ptr(),
                                       b["kt"].data_ptr(), b["vt"].data_ptr(), ts, hs, ws.data_ptr(), sh), "prepare")

        mark(0)
        check(N.nomas_kv_append(cache.handle, b["pk"].data_ptr(), b["pv"].data_ptr(), b["pk"].stride(0),
                                b["pk"].stride(1), n_frames_prev, 0, 0, 0, sh), "append")
        mark(1)
        check(N.nomas_mask_build(cache.handle, seg, 0, 0.25, 0, 0, ts, hs, mbuf_d.data_ptr(), sh), "mask dense")
        mark(2)
        prepare()
        mark(3)
        check(N.nomas_attn_run(cache.handle, seg, 0, 0.25, mbuf_d.data_ptr(), b["q"].data_ptr(), ts, hs, scale,
                               b["out_d"].data_ptr(), 0, ws.data_ptr(), sh), "attn dense")
        mark(4)
        check(N.nomas_mask_build(cache.handle, seg, 2, 0.25, 0, 0, ts, hs, mbuf_t.data_ptr(), sh), "mask text")
        mark(5)
        check(N.nomas_attn_run(cache.handle, seg, 2, 0.25, mbuf_t.data_ptr(), b["qt"].data_ptr(), ts, hs, scale,
                               b["out_t"].data_ptr(), 0, ws.data_ptr(), sh), "attn text")
        mark(6)
        check(N.nomas_mask_build(cache.handle, seg, 1, 0.25, b["q"].data_ptr(), b["kc"].data_ptr(), ts, hs,
                                 mbuf_s.data_ptr(), sh), "mask sparse")
        mark(7)
        check(N.nomas_attn_run(cache.handle, seg, 1, 0.25, mbuf_s.data_ptr(), b["q"].data_ptr(), ts, hs, scale,
                               b["out_s"].data_ptr(), 0, ws.data_ptr(), sh), "attn sparse")
        mark(8)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if cache.status() != 0:
        raise RuntimeError("device error during warm-up")
    st_now = cache.state()
    flops_dense = 4.0 * cfg.head_dim * cfg.heads * visible_key_sum(cfg, st_now["history_tokens"], st_now["head_tokens"])
    flops_text = 4.0 * cfg.head_dim * cfg.heads * text_key_sum(cfg, st_now["history_tokens"], st_now["head_tokens"])
    mv = mask_views(mbuf_s, lay_s)
    flops_sparse = 4.0 * cfg.head_dim * sparse_key_sum(mv["sel"], cfg, st_now["history_tokens"],
                                                       st_now["head_tokens"])
    append_bytes = (cfg.window_frames * cfg.tokens_per_frame) * cfg.heads * APPEND_BYTES_PER_TOKEN_HEAD(cfg.head_dim)
    prep_bytes = prepare_bytes(cfg, st_now["history_tokens"], st_now["head_tokens"])

    # timed region: K steps back to back, events on the launching stream
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with Clock(local_rank) as clk:
        t0.record(st)
        for _ in range(args.steps):
            step()
        t1.record(st)
        torch.cuda.synchronize()
    def reduce_max(x):
        tm = torch.tensor([x], device=dev)
        dist.all_reduce(tm, op=dist.ReduceOp.MAX)
        return float(tm.item())

    ms = t0.elapsed_time(t1)
    ms, _ = aggregate_ranks(ms, 0.0, world, reduce_max)
    if cache.status() != 0:
        raise RuntimeError("device error in the timed region")
    # per-phase breakdown: a separate pass of steps issued back to back with events between the
    # phases (no host synchronisation inside the pass, so no phase includes host launch latency)
    n_ph = max(3, min(args.steps, 10))
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(9)] for _ in range(n_ph)]
    for k in range(n_ph):
        step(evs[k])
    torch.cuda.synchronize()
    ph = [statistics.mean(evs[k][i].elapsed_time(evs[k][i + 1]) for k in range(n_ph)) for i in range(8)]

    # end to end: every step copies its inputs from pinned host memory, runs the same C-ABI calls and
    # copies both outputs back.  Like a serving loop, the copies of one step overlap the compute of
    # its neighbours: two device buffer sets, an H2D stream, the compute stream and a D2H stream,
    # ordered by events (inputs of set i are rewritten only after the compute that read them, outputs
    # of set i only after their D2H).  The timed region runs from before the first H2D copy to after
    # the last D2H copy.
    e2e = None
    if rank == 0 or world > 1:
        names = ("q", "kc", "vc", "kt", "vt", "qt", "pk", "pv")
        host = {n: bufs0[n].cpu().pin_memory() for n in names}
        bufs1 = {n: torch.empty_like(bufs0[n]) for n in names + ("out_d", "out_t", "out_s")}
        sets = [bufs0, bufs1]
        hout = [[torch.empty(bufs0[o].shape, dtype=torch.float32).pin_memory() for o in ("out_d", "out_t", "out_s")]
                for _ in range(2)]
        h2d = sum(t.numel() * t.element_size() for t in host.values())
        d2h = (2 * out_d.numel() + out_t.numel()) * 4
        s_h2d, s_d2h = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        done = [torch.cuda.Event() for _ in range(2)]
        ready = [torch.cuda.Event() for _ in range(2)]
        out_free = [torch.cuda.Event() for _ in range(2)]
        n_e2e = max(4, min(args.steps, 12))
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(s_h2d)
        for k in range(n_e2e):
            i = k % 2
            b = sets[i]
            if k >= 2:
                s_h2d.wait_event(done[i])          # step k-2 has finished reading set i
            with torch.cuda.stream(s_h2d):
                for n in names:
                    b[n].copy_(host[n], non_blocking=True)
            ready[i].record(s_h2d)
            st.wait_event(ready[i])
            if k >= 2:
                st.wait_event(out_free[i])         # the D2H of step k-2 has read set i's outputs
            step(b=b, stream=st)
            done[i].record(st)
            s_d2h.wait_event(done[i])
            with torch.cuda.stream(s_d2h):
                hout[i][0].copy_(b["out_d"], non_blocking=True)
                hout[i][1].copy_(b["out_t"], non_blocking=True)
                hout[i][2].copy_(b["out_s"], non_blocking=True)
            out_free[i].record(s_d2h)
        e1.record(s_d2h)
        torch.cuda.synchronize()
        ems, _ = aggregate_ranks(e0.elapsed_time(e1) / n_e2e, 0.0, world, reduce_max)   # slowest rank
        e2e = {"value": (flops_dense + flops_text + flops_sparse) / (ems * 1e-3) / 1e12 * world, "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ems, "steps": n_e2e,
               "pipelined": "H2D / compute / D2H on three streams, two buffer sets"}
    ws_bytes = {"production_1280x704": int(ws.numel())}
    del ws, mbuf_d, mbuf_s
    big = CONFIGS["C4"]
    c4 = KVCache.for_config(big, dev)
    ws_bytes["full_history_7th_of_7"] = int(N.nomas_attn_workspace_bytes(c4.handle, segment_text_of(big.current)))
    del c4
    linear = measure_linear(dev)
    return dict(ms=ms, phases=ph, flops_dense=flops_dense, flops_text=flops_text, flops_sparse=flops_sparse,
                append_bytes=append_bytes, linear=linear,
                prep_bytes=prep_bytes, ws_bytes=ws_bytes, clocks=clk.summary(), e2e=e2e, cfg=cfg)


def measure_linear(dev, reps=10):
    """The INT8-weight linear layer on the DiT's production shapes (tokens of one 30-frame 1280x704 segment
    plus its 1280 text tokens; hidden 2048, FFN 8192), synthetic bf16 activations and weights: the GEMM
    alone (nomas_linear_bf16 on the dequantised weights) and the whole call (dequantise + GEMM)."""
    import torch
    from int8_kv_cache_action_b200 import _nomas as N
    from int8_kv_cache_action_b200.runtime import Int8Linear
    out = {}
    for name, (m, k, n) in {"qkv_27680x2048x6144": (27680, 2048, 6144),
                            "ffn_down_27680x8192x2048": (27680, 8192, 2048)}.items():
        g = torch.Generator().manual_seed(77)
        x = (torch.randn(m, k, generator=g)).to(torch.bfloat16).to(dev)
        lin = Int8Linear.from_weights((torch.randn(n, k, generator=g) * 0.02).to(torch.bfloat16).to(dev))
        w = lin.dequantized()
        y = torch.empty((m, n), dtype=torch.bfloat16, device=dev)
        st = torch.cuda.current_stream().cuda_stream

        def gemm():
            N._check(N.nomas_linear_bf16(x.data_ptr(), m, k, k, w.data_ptr(), n, k, y.data_ptr(), n,
                                         N.NOMAS_DTYPE_BF16, lin.status_word.data_ptr(), st), "nomas_linear_bf16")

        def full():
            lin(x, out=y)

        res = {}
        for label, fn in (("gemm", gemm), ("w8a16", full)):
            for _ in range(3):
                fn()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            e0.record()
            for _ in range(reps):
                fn()
            e1.record()
            torch.cuda.synchronize()
            ms = e0.elapsed_time(e1) / reps
            res[label] = {"ms": ms, "tflops": 2.0 * m * n * k / (ms * 1e-3) / 1e12}
        if lin.status() != N.NOMAS_OK:
            raise RuntimeError("linear layer reported a device error")
        res["dequant_bytes"] = n * k * (1 + 2) + 4 * n
        out[name] = res
        del x, w, y, lin
    return out


def per_config(args):
    """One JSON line per config: the attention call (its mode: dense, or sparse for C3) and the mask
    build of that mode timed with CUDA events over back-to-back calls after 3 warm-ups, and the
    quantise-append of one 30-frame (C0: 2) segment into a fresh cache of the config's dimensions."""
    import torch
    from int8_kv_cache_action_b200 import _nomas as N
    from int8_kv_cache_action_b200.runtime import KVCache, mask_views, segment_text_of
    from int8_kv_cache_action_b200.workloads import CONFIGS, make_inputs, APPEND_BYTES_PER_TOKEN_HEAD
    dev = torch.device("cuda", 0)
    names = args.only.split(",") if args.only else ["C0", "C1", "C2", "C3", "C4"]
    for name in names:
        cfg = CONFIGS[name]
        inp = make_inputs(cfg)
        cache = KVCache.for_config(cfg, dev)
        for seg, kv in zip(cfg.prior, inp.prior):
            cache.append(kv.k.to(dev), kv.v.to(dev), seg.n_frames,
                         None if kv.head_k is None else kv.head_k.to(dev),
                         None if kv.head_v is None else kv.head_v.to(dev))
        seg = segment_text_of(cfg.current)
        q, kc, vc, kt, vt = (getattr(inp, n).to(dev) for n in ("q", "k_cur", "v_cur", "k_txt", "v_txt"))
        buf, lay = cache.build_mask(seg, cfg.mode, cfg.keep_frac, q, kc)
        ws = cache.workspace(seg)
        out = torch.empty((cfg.n_query, cfg.heads, cfg.head_dim), dtype=torch.float32, device=dev)
        st = cache.state()
        if cfg.mode:
            flops = 4.0 * cfg.head_dim * sparse_key_sum(mask_views(buf, lay)["sel"], cfg, st["history_tokens"],
                                                        st["head_tokens"])
        else:
            flops = 4.0 * cfg.head_dim * cfg.heads * visible_key_sum(cfg, st["history_tokens"], st["head_tokens"])

        def attn():
            cache.attention(seg, buf, q, kc, vc, kt, vt, mode=cfg.mode, keep_frac=cfg.keep_frac, workspace=ws,
                            out=out)

        reps = args.reps if args.reps else (10 if cfg.n_query > 1000 else 50)
        for _ in range(3):
            attn()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record()
        for _ in range(reps):
            attn()
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / reps
        # the mask build of the call's mode (sparse: block means, scores, ranking and lists)
        for _ in range(3):
            cache.build_mask(seg, cfg.mode, cfg.keep_frac, q, kc, mask_buf=buf)
        torch.cuda.synchronize()
        e0.record()
        for _ in range(reps):
            cache.build_mask(seg, cfg.mode, cfg.keep_frac, q, kc, mask_buf=buf)
        e1.record()
        torch.cuda.synchronize()
        mask_ms = e0.elapsed_time(e1) / reps
        status = cache.status()
        # append: the config's last prior segment (or the current segment's K/V) into a fresh cache
        src = inp.prior[-1] if cfg.prior else None
        k_app = (src.k if src is not None else inp.k_cur).to(dev)
        v_app = (src.v if src is not None else inp.v_cur).to(dev)
        nf = k_app.shape[0] // cfg.tokens_per_frame
        kept = min(nf, cfg.window_frames) if cfg.window_frames > 0 else nf
        fresh = [KVCache.for_config(cfg, dev) for _ in range(reps + 3)]
        for c in fresh[:3]:
            c.append(k_app, v_app, nf)
        torch.cuda.synchronize()
        e0.record()
        for c in fresh[3:]:
            c.append(k_app, v_app, nf)
        e1.record()
        torch.cuda.synchronize()
        app_ms = e0.elapsed_time(e1) / reps
        app_bytes = kept * cfg.tokens_per_frame * cfg.heads * APPEND_BYTES_PER_TOKEN_HEAD(cfg.head_dim)
        print(json.dumps({"config": name, "workload": cfg.name, "mode": "sparse" if cfg.mode else "dense",
                          "attn_ms": ms, "attn_tflops": flops / (ms * 1e-3) / 1e12, "attn_flops": flops,
                          "mask_ms": mask_ms,
                          "append_ms": app_ms, "append_gbs": app_bytes / (app_ms * 1e-3) / 1e9,
                          "append_kv_tokens_per_s": kept * cfg.tokens_per_frame * cfg.heads / (app_ms * 1e-3),
                          "status": status}), flush=True)
        del cache, fresh


_ORACLE_SETUP = None


def _oracle_setup():
    """Inputs of the workload and the oracle's cache after the prior segments (built once per process;
    not part of any timed region)."""
    global _ORACLE_SETUP
    if _ORACLE_SETUP is None:
        from int8_kv_cache_action_b200.workloads import CONFIGS, make_inputs
        from oracle.ring import OracleCache
        cfg = CONFIGS[WORKLOAD]
        inp = make_inputs(cfg)
        f = lambda t: t.float().numpy()
        oc = OracleCache(cfg.heads, cfg.head_dim, cfg.tokens_per_frame, cfg.window_frames, cfg.capacity_frames,
                         cfg.head_store_tokens)
        for seg, kv in zip(cfg.prior, inp.prior):
            oc.append(f(kv.k), f(kv.v), seg.n_frames)
        _ORACLE_SETUP = (cfg, oc, (f(inp.q), f(inp.k_cur), f(inp.v_cur), f(inp.k_txt), f(inp.v_txt)))
    return _ORACLE_SETUP


def cpu_oracle_sample(seconds_budget=15.0, rows_per_head_start=16):
    """Time the CPU oracle (as it stands) on a bounded sample of the same workload's dense attention."""
    import numpy as np
    from threadpoolctl import threadpool_info

    from oracle import attention as att

    cfg, oc, (qf, kcf, vcf, ktf, vtf) = _oracle_setup()
    rng = np.random.default_rng(0)
    n = rows_per_head_start
    while True:
        rows = np.sort(rng.choice(cfg.n_query, n, replace=False))
        t0 = time.perf_counter()
        att.attention(oc, qf, kcf, vcf, ktf, vtf, cfg.current, 1.0 / math.sqrt(cfg.head_dim), rows=rows)
        dt = time.perf_counter() - t0
        if dt > seconds_budget / 4 or n >= cfg.n_query:
            break
        n = min(cfg.n_query, n * 4)
    vis = 15840 + 26400 + 768
    T = cfg.tokens_per_frame
    flops = 0.0
    for r in rows:
        t = r // T
        flops += 4.0 * cfg.head_dim * cfg.heads * (vis + sum(a.len for a in cfg.current.tails if a.f0 <= t < a.f1))
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
            "sample": f"dense attention of {len(rows)} random query rows x 16 heads of the production shape "
                      f"(fp64 numpy oracle, {dt:.1f} s)"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--per-config", action="store_true",
                    help="print one line per config (attention call and append) instead of the step line")
    ap.add_argument("--only", default="", help="with --per-config: comma-separated config names (C0..C4, C3r)")
    ap.add_argument("--reps", type=int, default=0, help="with --per-config: timed calls per config")
    ap.add_argument("--attn-kernel", type=int, default=0,
                    help="head_dim-128 attention kernel: 0 chosen per call, 1 one query block per CTA, 2 block pairs")
    ap.add_argument("--linear-only", action="store_true",
                    help="print one line with the INT8-weight linear layer on the DiT shapes only")
    args = ap.parse_args()
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    pk, pk_kind = peaks()

    if args.impl == "reference":
        if rank != 0:
            return
        from int8_kv_cache_action_b200.workloads import CONFIGS
        vals = []
        for i in range(args.warmup + args.steps):
            r = cpu_oracle_sample(seconds_budget=6.0)
            if i >= args.warmup:
                vals.append(r)
        v = statistics.mean(x["value"] for x in vals)
        line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOP/s", "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": step_config(CONFIGS[WORKLOAD], args.gpus),
                "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": vals[0]["cores"], "kind": "oracle",
                                 "sample": vals[0]["sample"]},
                "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return

    if args.attn_kernel:
        from int8_kv_cache_action_b200 import _nomas as N
        N.nomas_set_attn_kernel(args.attn_kernel)
    if args.per_config:
        per_config(args)
        return
    if args.linear_only:
        import torch
        lin = measure_linear(torch.device("cuda", 0), reps=args.reps or 10)
        peak = pk.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
        print(json.dumps({"linear": lin, "peak_bf16_tflops": peak, "peak_kind": pk_kind,
                          "frac": {k: v["gemm"]["tflops"] / peak for k, v in lin.items()}}))
        return

    import torch
    import torch.distributed as dist
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    cpu_base = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu_base = cpu_oracle_sample()
    r = run_ours(args, rank, world, local_rank)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    cfg = r["cfg"]
    ms_step = r["ms"] / args.steps
    flops = r["flops_dense"] + r["flops_text"] + r["flops_sparse"]
    _, value = aggregate_ranks(ms_step, flops, world)
    value /= 1e12
    # append, mask dense, prepare, run dense, mask text, run text, mask sparse, run sparse
    ph = r["phases"]
    dense_tflops = r["flops_dense"] / (ph[3] * 1e-3) / 1e12
    text_tflops = r["flops_text"] / (ph[5] * 1e-3) / 1e12
    sparse_tflops = r["flops_sparse"] / (ph[7] * 1e-3) / 1e12
    dense_call_tflops = r["flops_dense"] / ((ph[2] + ph[3]) * 1e-3) / 1e12
    sparse_call_tflops = r["flops_sparse"] / (ph[7] * 1e-3) / 1e12   # the workspace is already prepared
    append_gbs = r["append_bytes"] / (ph[0] * 1e-3) / 1e9
    prep_ms = ph[2]
    prep_gbs = r["prep_bytes"] / (prep_ms * 1e-3) / 1e9
    peak_sus = pk.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    peak_burst = pk.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    hbm = pk.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    traffic = measured_traffic("attn")
    append_traffic = measured_traffic("append")
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": step_config(cfg, world),
        "roofline": {"bound": "tensor",
                     "kernel": "attn_pair_kernel (nomas_attn_run, dense: one CTA per query-block pair)",
                     "achieved": dense_tflops,
                     "peak": peak_burst, "unit": "TFLOP/s", "frac": dense_tflops / peak_burst,
                     "peak_kind": f"bf16 dense, burst ({pk_kind}): the kernel runs {ph[3]:.2f} ms at a time",
                     "frac_of_sustained": dense_tflops / peak_sus, "traffic": traffic},
        "roofline_append": {"bound": "hbm", "kernel": "quant_append_kernel<128>", "achieved": append_gbs,
                            "peak": hbm, "unit": "GB/s", "frac": append_gbs / hbm, "traffic": append_traffic,
                            "peak_kind": f"HBM copy ({pk_kind})"},
        "roofline_dequant": {"bound": "hbm",
                             "kernel": "nomas_attn_prepare (prepare_kernel: INT8 history codes "
                                       "and bf16 current/text K,V widened to fp16)",
                             "achieved": prep_gbs, "peak": hbm, "unit": "GB/s", "frac": prep_gbs / hbm,
                             "bytes_per_call": r["prep_bytes"], "ms_per_call": prep_ms,
                             "traffic": measured_traffic("prepare")},
        "breakdown_ms": {"append": ph[0], "mask_dense": ph[1], "prepare_dense": ph[2], "attn_dense": ph[3],
                         "mask_text": ph[4], "attn_text": ph[5], "mask_sparse": ph[6], "attn_sparse": ph[7]},
        "attn_text_tflops": text_tflops,
        "attn_dense_tflops": dense_tflops, "attn_sparse_tflops": sparse_tflops,
        "attn_dense_call_tflops": dense_call_tflops, "attn_sparse_call_tflops": sparse_call_tflops,
        "attn_workspace_bytes": r["ws_bytes"],
        "roofline_linear": {
            "bound": "tensor", "kernel": "gemm2_bf16_kernel (nomas_linear_bf16; nomas_w8a16_linear adds the dequantise "
                                        "pre-pass)",
            "peak": peak_burst, "unit": "TFLOP/s", "peak_kind": f"bf16 dense, burst ({pk_kind})",
            "shapes": {k: {"gemm_tflops": v["gemm"]["tflops"], "gemm_frac": v["gemm"]["tflops"] / peak_burst,
                           "gemm_ms": v["gemm"]["ms"], "w8a16_ms": v["w8a16"]["ms"],
                           "w8a16_tflops": v["w8a16"]["tflops"]} for k, v in r["linear"].items()},
            "traffic_qkv": measured_traffic("linear"),
            "timed": "outside the step (the step is the attention path)"},
        "flops_per_step": {"dense": r["flops_dense"], "text": r["flops_text"], "sparse": r["flops_sparse"]},
        "kv_tokens_per_s_append": (cfg.window_frames * cfg.tokens_per_frame) * cfg.heads / (ph[0] * 1e-3),
        "cpu_baseline": cpu_base,
        "e2e": r["e2e"],
        "gpu_launches": (LAUNCHES_PER_STEP - 1 + dense_attention_launches(
            cfg.n_query, cfg.heads, torch.cuda.get_device_properties(local_rank).multi_processor_count)) * args.steps,
        "clocks": r["clocks"],
    }
    print(json.dumps(line))


if __name__ == "__main__":
    main()
