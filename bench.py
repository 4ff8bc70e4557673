#!/usr/bin/env python
"""Benchmark of the MAC-Attention decode step on B200.

A step is one mac_decode_step (match + amend/complete/miss + merge) over all
B sequences of one attention layer, on the 128K-context workload
(B=4, 32 query / 8 KV heads, D=128, bf16 contiguous KV, W=32, band=256, 90%
of queries near-repeats of a recent one).  Inputs are seeded synthetic data of
that shape (synth.WORKLOADS["long_128k"]).  L2 is flushed (256 MiB write)
between timed steps.

Prints one JSON line (rank 0).  Multi-GPU (torchrun): every rank runs its own
batch of the workload (independent problems, no collective on the data path),
so scaling is weak and value = all ranks' steps / max-over-ranks time.

--impl reference times the fp64 CPU oracle on the host cores instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "MAC decode-attention steps/s at 128K ctx"
UNIT = "steps/s"
L2_FLUSH_BYTES = 256 << 20


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def _kernel_hash() -> str:
    """Hash of the step kernel's source code (the attention file, the match
    stage and device helpers it includes and the shared layout; comments and
    blank space removed, so that a comment edit does not orphan a profile)."""
    h = hashlib.sha256()
    for f in ("mac_attend.cu", "mac_attend_dev.cuh", "mac_internal.cuh", "mac_match_dev.cuh"):
        with open(os.path.join(ROOT, "kv_cache_reuse_b200", "csrc", f)) as fh:
            src = fh.read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        src = re.sub(r"//[^\n]*", "", src)
        h.update("".join(src.split()).encode())
    return h.hexdigest()[:16]


def _profiled_traffic():
    """Ratio of DRAM bytes to algorithmic bytes of the step kernel from the
    committed ncu summary, if it was taken on the current kernel source (else None)."""
    p = os.path.join(ROOT, "profiles", "mac_step_long_128k_traffic.txt")
    try:
        txt = open(p).read()
    except OSError:
        return None
    m = re.search(r"kernel_source_sha256_16:\s*([0-9a-f]+)", txt)
    b = re.search(r"dram_traffic_over_algorithmic:\s*([0-9.eE+]+)", txt)
    if not m or not b or m.group(1) != _kernel_hash():
        return None
    return float(b.group(1))


class ClockSampler:
    """Samples SM clock and clock-event reasons with NVML during the timed region."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, index: int):
        self.samples, self.reasons, self.ok = [], 0, False
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            pass
        self._stop = threading.Event()

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reasons |= int(self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h))
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        return {"sm_mhz": float(np.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": [n for b, n in self.REASONS.items() if self.reasons & b],
                "samples": len(self.samples)}


_BAD_REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown")


def clocks_rejected(c) -> bool:
    """A timed region whose clock record disqualifies it: a hardware or
    thermal slowdown, or SM clocks well below their maximum with no reason
    reported (a clock lock left behind).  A power cap alone is kept."""
    if any(r in c.get("reasons", []) for r in _BAD_REASONS):
        return True
    mhz, mx = c.get("sm_mhz"), c.get("sm_max_mhz")
    return bool(mhz and mx and mhz < 0.85 * mx and not c.get("reasons"))


def step_bytes(wl, hit, mpos, seq_lens, occ, qes=4, res=4):
    """Algorithmic HBM bytes of one step: (match kernel, attention kernel, K/V only).

    hit, mpos: [B][Hkv] decisions, or [B][Hq] with per-head matching.  qes, res:
    bytes of a query element and of a window element (q and stored o).
    Match: query G*D*qes per unit, window scan occ*G*D*res, ring-q write
    G*D*res, rotated query write G*D*4.  Attention: K+V of every key attended
    fresh -- the union of the unit's heads' ranges -- (2*D*2 per key), rotated
    query G*D*4, reused state (D*res + 8) per reusing head, new state
    G*(D*res + 8) + position, out and lse G*(D+1)*4.
    """
    G, D, band = wl.G, wl.D, wl.band
    hpd = G * wl.Hkv // hit.shape[1]  # heads per decision
    gd = G * D
    kv = att = mt = 0
    for b in range(wl.B):
        p_t = int(seq_lens[b]) - 1
        for h in range(wl.Hkv):
            dec = range(h * G // hpd, (h + 1) * G // hpd)
            start = min(max(0, int(mpos[b, d]) - band) if hit[b, d] else 0 for d in dec)
            reusing = sum(hpd for d in dec if hit[b, d])
            keys = p_t + 1 - start
            kv += keys * 2 * D * 2
            att += gd * 4 + reusing * (D * res + 8) + G * (D * res + 8) + 4 + G * (D + 1) * 4
            mt += gd * qes + occ * gd * res + gd * res + gd * 4
    return mt, att + kv, kv


def rank_workload(args, rank):
    """The workload one rank runs: every rank takes its own batch (its own seed),
    so ranks share no data and the job scales weakly with no collective."""
    base = synth.WORKLOADS[args.workload]
    if args.batch:
        base = base.with_(B=args.batch, L0=base.L0[:1] * args.batch)
    if args.tau is not None:
        base = base.with_(tau=args.tau)
    hq, hkv = getattr(args, "q_heads", 0), getattr(args, "kv_heads", 0)
    if hq or hkv:
        base = base.with_(Hq=hq or base.Hq, Hkv=hkv or base.Hkv)
    return base, base.with_(seed=base.seed + 1000 * rank)


def bench_config(wl, paged: bool, world: int) -> dict:
    """The workload description both arms print (same keys, same values)."""
    return {"workload": wl.name, "batch": wl.B, "q_heads": wl.Hq, "kv_heads": wl.Hkv, "head_dim": wl.D,
            "context": int(wl.L0[0]), "window": wl.W, "band": wl.band, "tau": wl.tau,
            "hit_label_rate": wl.hit_model[1], "kv": "bf16 %s" % ("paged" if paged else "contiguous"),
            "l2": "flushed between timed steps (256 MiB write)", "parallelism": "replicas" if world > 1 else "1 GPU"}


def max_over_ranks(x: float, world: int, device) -> float:
    """Largest value of x over the ranks (the job's time is its slowest rank's)."""
    if world <= 1:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def run_mac(args, rank, world, local_rank):
    import torch
    import kv_cache_reuse_b200 as mac

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    base, wl = rank_workload(args, rank)
    T = max(base.steps, args.warmup + args.steps)
    stream = synth.queries(wl, T)
    cache = synth.kv_cache(wl, T)
    K = torch.from_numpy(cache.K.view(np.int16)).to(dev)
    V = torch.from_numpy(cache.V.view(np.int16)).to(dev)
    bt = None if not cache.paged else torch.from_numpy(cache.block_table).to(dev)
    kw = dict(max_pages_per_seq=cache.block_table.shape[1], num_pages=cache.num_pages) if cache.paged else \
        dict(capacity=cache.max_seq)
    B, Hq, Hkv, D = wl.B, wl.Hq, wl.Hkv, wl.D
    q_all = torch.from_numpy(stream.q).to(dev)
    pos_all = torch.from_numpy(stream.rope_pos).to(dev)
    lens_all = torch.from_numpy(stream.seq_lens).to(dev)
    out = torch.empty((B, Hq, D), dtype=torch.float32, device=dev)
    lse = torch.empty((B, Hq), dtype=torch.float32, device=dev)
    hit_all = torch.zeros((T, B, Hq), dtype=torch.uint8, device=dev)  # [B][Hkv] used unless per-head
    mpos_all = torch.zeros((T, B, Hq), dtype=torch.int32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    s = torch.cuda.current_stream(dev)
    peak, peak_kind = _peaks()

    sptr = s.cuda_stream
    hsz = (B, Hkv)

    # the stream the timed steps read (the bf16, per-head, hit-path and context runs swap it)
    cur = {"q": q_all, "pos": pos_all, "lens": lens_all, "stream": stream}

    def ptrs(t):
        return (cur["q"][t].data_ptr(), cur["pos"][t].data_ptr(), cur["lens"][t].data_ptr(), hit_all[t].data_ptr(),
                mpos_all[t].data_ptr())

    def timed_run(tau, nwarm, nsteps, split, cfg=None, bytes_stream=None):
        """Warm-up, then nsteps timed steps.  split=False: one mac_decode_step per
        step (match and attend back to back, programmatic launch), events around
        the step.  split=True: events also between the two kernels, for the
        per-kernel roofline.  The timed steps are queued behind a GPU sleep so the
        host stays ahead of the device and no host latency enters the events."""
        cfg = dict(cfg or {})
        one_launch = cfg.pop("one_launch", 1)
        st = mac.MacState.for_workload(wl, tau=tau, **kw, **cfg)
        mac.mac_set_one_launch(st, one_launch)
        h = st.handle
        nd = Hq if cfg.get("match_per_head") else Hkv  # decisions per sequence
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
               torch.cuda.Event(enable_timing=True)) for _ in range(nsteps)]
        Kp, Vp, btp, outp, lsep = K.data_ptr(), V.data_ptr(), (bt.data_ptr() if bt is not None else None), \
            out.data_ptr(), lse.data_ptr()
        for t in range(nwarm):
            q, pz, ln, hm, mp = ptrs(t)
            mac.mac_decode_step(h, q, pz, Kp, Vp, btp, ln, outp, lsep, hm, mp, sptr)
            flush.zero_()
        torch.cuda.synchronize(dev)
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize(dev)
        pre = [ptrs(nwarm + i) for i in range(nsteps)]
        clocks = ClockSampler(local_rank)
        with clocks:
            torch.cuda._sleep(int(2e6 + 4e5 * nsteps))  # GPU cycles; lets the host enqueue ahead
            for i in range(nsteps):
                q, pz, ln, hm, mp = pre[i]
                e0, e1, e2 = ev[i]
                e0.record(s)
                if split:
                    mac.mac_match(h, q, pz, btp, ln, outp, lsep, hm, mp, sptr)
                    e1.record(s)
                    mac.mac_attend(h, Kp, Vp, btp, outp, lsep, sptr)
                else:
                    mac.mac_decode_step(h, q, pz, Kp, Vp, btp, ln, outp, lsep, hm, mp, sptr)
                e2.record(s)
                flush.zero_()
            torch.cuda.synchronize(dev)
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize(dev)
        status = st.get_status()
        one = mac.mac_one_launch(st) if not split else 0
        st.close()
        step_ms = [a.elapsed_time(c) for a, b_, c in ev]
        att_ms = [b_.elapsed_time(c) for a, b_, c in ev] if split else [0.0] * nsteps
        match_ms = [a.elapsed_time(b_) for a, b_, c in ev] if split else [0.0] * nsteps
        # decisions of a step: the first nd entries of each step's buffer, [B][nd]
        hits = hit_all.view(T, -1)[nwarm:nwarm + nsteps, :B * nd].reshape(nsteps, B, nd).cpu().numpy()
        mpos = mpos_all.view(T, -1)[nwarm:nwarm + nsteps, :B * nd].reshape(nsteps, B, nd).cpu().numpy()
        qes = 2 if cfg.get("q_bf16") else 4
        res_ = 2 if cfg.get("ring_bf16") else 4
        mt_b = at_b = kv_b = dense_b = 0
        for i in range(nsteps):
            t = nwarm + i
            occ = min(t, wl.W)
            a, b_, c = step_bytes(wl, hits[i], mpos[i], cur["stream"].seq_lens[t], occ, qes, res_)
            mt_b += a
            at_b += b_
            kv_b += c
            dense_b += synth.dense_equiv_kv_bytes(wl, cur["stream"].seq_lens[t])
        tot_ms = float(np.sum(step_ms))
        allhit = [bool(hits[i].all()) for i in range(nsteps)]
        by_class = {k: (float(np.mean([step_ms[i] for i in range(nsteps) if allhit[i] == v])) * 1e3
                        if any(allhit[i] == v for i in range(nsteps)) else None)
                    for k, v in (("all_hit_us", True), ("with_miss_us", False))}
        by_class["with_miss_steps"] = int(nsteps - sum(allhit))
        return dict(total_ms=tot_ms, step_ms=step_ms, att_ms=float(np.sum(att_ms)), match_ms=float(np.sum(match_ms)),
                    one_launch=one, by_class=by_class,
                    att_bytes=at_b, match_bytes=mt_b, kv_bytes=kv_b, dense_bytes=dense_b,
                    hit_frac=float(hits.mean()), status=status, clocks=clocks.summary())

    main = timed_run(wl.tau, args.warmup, args.steps, split=False)
    # a disqualified clock record on any rank: every rank measures once more
    remeasured = max_over_ranks(1.0 if clocks_rejected(main["clocks"]) else 0.0, world, dev) > 0
    if remeasured:
        main = timed_run(wl.tau, args.warmup, args.steps, split=False)
    main["clocks"]["remeasured"] = remeasured
    kern = timed_run(wl.tau, args.warmup, args.steps, split=True)
    # the same steps as two launches (match kernel, then attention kernel with
    # programmatic dependent launch), timed as the main run is
    main2 = timed_run(wl.tau, args.warmup, args.steps, split=False, cfg={"one_launch": 0})
    allmiss = allmiss2 = None
    if args.miss_steps > 0:
        nm = min(args.miss_steps, T - 3)
        allmiss = timed_run(0.0, 3, nm, split=False)   # the step as it runs (one launch where it applies)
        allmiss2 = timed_run(0.0, 3, nm, split=True)   # the two kernels timed apart
    warm = None
    if args.warm_start:
        # seed the windows from the first W positions of the stream (as prefill
        # positions): W threshold-0 steps over the whole prefix of every unit
        n = min(wl.W, T)
        st = mac.MacState.for_workload(wl, **kw)
        args_w = (n, q_all[:n].contiguous(), pos_all[:n].contiguous(), K, V, bt, lens_all[:n].contiguous())
        mac.mac_warm_start(st, *args_w, stream=s)  # warm-up
        flush.zero_()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s)
        mac.mac_warm_start(st, *args_w, stream=s)
        e1.record(s)
        torch.cuda.synchronize(dev)
        wms = e0.elapsed_time(e1)
        wbytes = sum(int(stream.seq_lens[j][b]) * 2 * wl.D * 2 * wl.Hkv for j in range(n) for b in range(wl.B))
        warm = {"positions": n, "ms": wms, "kv_bytes": wbytes, "gbs": wbytes / (wms * 1e-3) / 1e9,
                "frac": wbytes / (wms * 1e-3) / 1e9 / peak, "device_status": st.get_status()}
        st.close()
    layers = run_layers(args, wl, stream, cache, K, V, bt, kw, dev, peak) if args.layers > 0 else None
    bf16 = None
    if not args.no_bf16:
        # bf16 queries and bf16 window: the same stream with its queries rounded to bf16
        cur["q"] = torch.from_numpy(synth.f32_to_bf16_bits(stream.q).view(np.int16)).to(dev)
        cfg = {"q_bf16": 1, "ring_bf16": 1}
        bf16 = (timed_run(wl.tau, args.warmup, args.steps, split=False, cfg=cfg),
                timed_run(wl.tau, args.warmup, args.steps, split=True, cfg=cfg))
        cur["q"] = q_all
    perhead = None
    if not args.no_per_head:
        # per-head matching on a stream whose query heads repeat on their own
        wh = wl.with_(head_labels=True)
        cur["q"] = torch.from_numpy(synth.queries(wh, T).q).to(dev)
        cfg = {"match_per_head": 1}
        perhead = (timed_run(wl.tau, args.warmup, args.steps, split=False, cfg=cfg),
                   timed_run(wl.tau, args.warmup, args.steps, split=True, cfg=cfg))
        cur["q"] = q_all
    hitrun = hitrun2 = None
    hitctx = []
    if args.hit_steps > 0:
        # the hit path alone: the same shape with every labelled step a near-repeat
        qh = synth.queries(wl.with_(hit_model=("iid", 1.0)), T).q
        cur["q"] = torch.from_numpy(qh).to(dev)
        # the windows filled first (W untimed steps), so every timed step scans a full window
        hitrun = timed_run(wl.tau, wl.W, min(args.hit_steps, T - wl.W), split=False)
        hitrun2 = timed_run(wl.tau, wl.W, min(args.hit_steps, T - wl.W), split=True)
        cur["q"] = q_all
        if not cache.paged:
            # the same hit stream at shorter contexts, on the same cache: a hit's
            # cost should not depend on the context length
            for L in (8192, 32768):
                sc = synth.queries(wl.with_(hit_model=("iid", 1.0), L0=(L,) * B), T)
                cur.update(q=torch.from_numpy(sc.q).to(dev), pos=torch.from_numpy(sc.rope_pos).to(dev),
                           lens=torch.from_numpy(sc.seq_lens).to(dev), stream=sc)
                r = timed_run(wl.tau, wl.W, min(args.hit_steps, T - wl.W), split=False)
                hitctx.append((L, r))
            cur.update(q=q_all, pos=pos_all, lens=lens_all, stream=stream)
            hitctx.append((int(wl.L0[0]), hitrun))

    quality = None
    if not args.no_quality:
        quality = run_quality(args, wl, stream, K, V, bt, kw, dev)
        quality["identity_rope"] = run_quality(args, wl, stream, K, V, bt, kw, dev, identity_rope=True)
        quality["note"] = ("a hit reuses prefix attention computed with the matched query rotated to its own "
                           "position; on structure-free random queries and keys every RoPE frequency weighs the "
                           "same, so the position shift alone decorrelates the reused scores (compare identity_rope)")

    # max over ranks of the timed duration
    tot = max_over_ranks(main["total_ms"], world, dev)

    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, wl, stream, cache, K, V, bt, kw, dev, world)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = run_cpu_baseline(wl, stream, cache, args.cpu_seconds)

    mqa = None
    if args.mqa_steps > 0:
        # multi-query groups: the workload's shape with 32 query heads over one KV
        # head, every step a miss (the dense-decode bandwidth of the chunked
        # kernel) and the workload's own repeat stream
        wq = wl.with_(Hq=32, Hkv=1)
        mqa = {"all_miss": run_shape(wq.with_(tau=0.0), args.mqa_steps, dev, peak, nwarm=3),
               "mixed": run_shape(wq, args.mqa_steps, dev, peak)}
    traces = None
    if args.trace_steps > 0:
        # the phase breakdown of hit steps (and of steps with misses) from the device trace
        traces = {"long_128k_all_hit": run_trace(wl.with_(hit_model=("iid", 1.0)), args.trace_steps, dev, peak),
                  "long_128k_mixed": run_trace(wl, args.trace_steps, dev, peak),
                  "paged_mixed_all_hit": run_trace(synth.WORKLOADS["paged_mixed"].with_(hit_model=("iid", 1.0)),
                                                   args.trace_steps, dev, peak),
                  "mqa_32_1_all_miss": run_trace(wl.with_(Hq=32, Hkv=1, tau=0.0), 4, dev, peak)}
    paged_gap = None
    if args.miss_steps > 0 and args.paged_gap:
        # paged against contiguous K/V at the same size, every step a miss: the
        # paged_mixed shape (16 sequences of 8K-64K keys) in both layouts
        wp = synth.WORKLOADS["paged_mixed"].with_(tau=0.0)
        paged_gap = {"paged": run_shape(wp, 4, dev, peak, nwarm=3),
                     "contiguous": run_shape(wp.with_(page_size=0), 4, dev, peak, nwarm=3)}
    hitshapes = []
    if args.hit_steps > 0 and args.hit_shapes:
        hitshapes = [run_hit_shape(n, args.hit_steps, dev, peak, world) for n in args.hit_shapes.split(",") if n]

    if rank != 0:
        return None
    K_ = args.steps
    gbs = lambda nbytes, ms: nbytes / (ms * 1e-3) / 1e9

    def two_launch(r, n):
        """The same steps with the match and attention kernels launched (and timed) apart."""
        a, m = gbs(r["att_bytes"], r["att_ms"]), gbs(r["match_bytes"], r["match_ms"])
        return {"attend": {"kernel": "mac_attend_kernel", "achieved": a, "frac": a / peak,
                           "mb_per_launch": r["att_bytes"] / n / 1e6, "us_per_launch": r["att_ms"] * 1e3 / n},
                "match": {"kernel": "mac_match_kernel", "achieved": m, "frac": m / peak,
                          "mb_per_launch": r["match_bytes"] / n / 1e6, "us_per_launch": r["match_ms"] * 1e3 / n},
                "step_us": r["total_ms"] * 1e3 / n}

    def brief(t):
        """A two-launch record as it goes on the one JSON line (the full one on stderr)."""
        return {"attend_frac": t["attend"]["frac"], "attend_us": t["attend"]["us_per_launch"],
                "match_us": t["match"]["us_per_launch"], "step_us": t["step_us"]}

    def step_roof(r, n):
        """The step as it runs: one launch (match, whole units, split ranges) or two."""
        nbytes = r["att_bytes"] + r["match_bytes"]
        a = gbs(nbytes, r["total_ms"])
        return {"kernel": "mac_step_kernel" if r["one_launch"] else "mac_match_kernel + mac_attend_kernel",
                "achieved": a, "frac": a / peak, "mb_per_launch": nbytes / n / 1e6,
                "us_per_launch": r["total_ms"] * 1e3 / n}

    occ = [min(t, wl.W) for t in range(args.warmup, args.warmup + K_)]
    main_roof = step_roof(main, K_)
    roof = {"bound": "hbm", "kernel": main_roof["kernel"], "achieved": main_roof["achieved"], "peak": peak,
            "peak_kind": peak_kind, "unit": "GB/s", "frac": main_roof["frac"],
            # traffic of the step kernel from the committed ncu capture, when it matches this source
            "traffic": (_profiled_traffic() * (main["att_bytes"] + main["match_bytes"]) / K_)
            if _profiled_traffic() else None,
            "bytes_per_launch": (main["att_bytes"] + main["match_bytes"]) / K_,
            "us_per_launch": main["total_ms"] * 1e3 / K_,
            "by_class": main["by_class"],
            "two_launch": dict(brief(two_launch(kern, K_)), steps_per_s=K_ / (main2["total_ms"] * 1e-3),
                               step_us_back_to_back=main2["total_ms"] * 1e3 / K_, by_class=main2["by_class"])}
    detail = {"two_launch": two_launch(kern, K_)}
    if allmiss:
        n = len(allmiss["step_ms"])
        roof["miss"] = dict(step_roof(allmiss, n),
                            workload="%s, threshold 0 (every unit misses)" % wl.name,
                            steps_per_s=n / (allmiss["total_ms"] * 1e-3),
                            two_launch=brief(two_launch(allmiss2, n)))
        detail["all_miss"] = {"steps": n, "ms_per_step": allmiss["total_ms"] / n, "two_launch": two_launch(allmiss2, n),
                              "speedup_of_mac": (world * K_ / (tot * 1e-3)) / (n / (allmiss["total_ms"] * 1e-3)),
                              "clocks": allmiss["clocks"]}
    if hitrun:
        n = len(hitrun["step_ms"])
        roof["hit"] = dict(step_roof(hitrun, n), workload="%s, every step a repeat" % wl.name,
                           hit_fraction=hitrun["hit_frac"], two_launch=brief(two_launch(hitrun2, n)),
                           larger={h["workload"].split(" ")[0]: {"step_us": h["step"]["us"], "step_frac": h["step"]["frac"]}
                                   for h in hitshapes})
        detail["hit_path"] = {"steps": n, "clocks": hitrun["clocks"], "shapes": hitshapes,
                              "two_launch": two_launch(hitrun2, n)}
        if hitctx:
            # step time of the same all-hit stream against the context length (the same MB per step)
            roof["hit"]["us_vs_context"] = {str(L): r["total_ms"] * 1e3 / len(r["step_ms"]) for L, r in hitctx}
            detail["hit_path"]["vs_context"] = [
                {"context": L, "step_us": r["total_ms"] * 1e3 / len(r["step_ms"]),
                 "step_mb": (r["att_bytes"] + r["match_bytes"]) / len(r["step_ms"]) / 1e6} for L, r in hitctx]
    if paged_gap:
        roof.setdefault("miss", {})["paged_vs_contiguous"] = {  # the paged_mixed shape, every unit missing
            "paged_frac": paged_gap["paged"]["step"]["frac"], "contiguous_frac": paged_gap["contiguous"]["step"]["frac"],
            "paged_attend_frac": paged_gap["paged"]["attend"]["frac"],
            "contiguous_attend_frac": paged_gap["contiguous"]["attend"]["frac"]}
        detail["paged_vs_contiguous"] = paged_gap
    if mqa:
        a = mqa["all_miss"]["attend"]
        roof.setdefault("miss", {})["mqa_32_1"] = {"frac": a["frac"], "us_per_launch": a["us_per_launch"]}
        detail["mqa_32_1"] = mqa
    res = {
        "metric": METRIC, "value": world * K_ / (tot * 1e-3), "unit": UNIT, "n_gpus": world, "steps": K_,
        "warmup": args.warmup, "ms_per_step": tot / K_, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": bench_config(wl, cache.paged, world),
        "roofline": roof,
        "hit_fraction": main["hit_frac"],
        "window_occupancy": {"mean": float(np.mean(occ)), "min": int(min(occ)), "max": int(max(occ)),
                             "window": wl.W},
        "gpu_launches": (1 if main["one_launch"] else 2) * K_ * world,
        "clocks": main["clocks"],
        "device_status": main["status"],
    }
    if layers:
        res["layer_stack"] = {k: layers[k] for k in ("layers", "us_per_layer", "tokens_per_s", "hit_fraction",
                                                    "device_status")}
        detail["layer_stack"] = layers
    if e2e:
        res["e2e"] = e2e
    if cpu:
        res["cpu_baseline"] = cpu
    detail.update({
        "kernel_ms_per_step_two_launch": {"match": kern["match_ms"] / K_, "attend": kern["att_ms"] / K_,
                                          "timed_separately": kern["total_ms"] / K_},
        "step_gbs": (main["att_bytes"] + main["match_bytes"]) / (main["total_ms"] * 1e-3) / 1e9,
        "effective_kv_gbs": main["dense_bytes"] / (main["total_ms"] * 1e-3) / 1e9,
        "kv_bytes_per_step": main["kv_bytes"] / K_, "dense_kv_bytes_per_step": main["dense_bytes"] / K_,
        "timing": "CUDA events around each step on the launching stream; steps queued behind a GPU sleep so host "
                  "latency is excluded; roofline from a second timed pass with events between the two kernels"})
    for name, pair, what in (("bf16_window", bf16, {"q": "bf16", "window_q_and_o": "bf16"}),
                             ("per_head", perhead, {"matching": "per query head",
                                                    "stream": "each query head repeats a recent query of its own "
                                                              "(rate as the workload) or draws fresh"})):
        if not pair:
            continue
        run, kr = pair
        a_gbs = kr["att_bytes"] / (kr["att_ms"] * 1e-3) / 1e9
        detail[name] = dict(what, **{
            "steps_per_s": K_ / (run["total_ms"] * 1e-3), "ms_per_step": run["total_ms"] / K_,
            "vs_headline": (K_ / (run["total_ms"] * 1e-3)) / (world * K_ / (tot * 1e-3)),
            "hit_fraction": run["hit_frac"], "match_ms_per_step": kr["match_ms"] / K_,
            "attend_ms_per_step": kr["att_ms"] / K_, "match_bytes_per_step": kr["match_bytes"] / K_,
            "attend_bytes_per_step": kr["att_bytes"] / K_, "attend_gbs": a_gbs, "attend_frac": a_gbs / peak,
            "match_gbs": kr["match_bytes"] / (kr["match_ms"] * 1e-3) / 1e9,
            "clocks": run["clocks"], "device_status": run["status"]})
    if quality:
        detail["approximation_vs_dense"] = quality
    if traces:
        detail["phase_trace"] = traces
    if warm:
        detail["warm_start"] = warm
    res["detail"] = "full record on stderr (one JSON line)"
    return res, detail


def run_hit_shape(name, nsteps, dev, peak, world):
    """The hit path alone on another workload's shape: every labelled step a
    near-repeat of a recent query."""
    r = run_shape(synth.WORKLOADS[name].with_(hit_model=("iid", 1.0)), nsteps, dev, peak)
    r["workload"] = "%s shape, every step a repeat" % name
    return r


def run_shape(wl, nsteps, dev, peak, nwarm=None):
    """Steps of another workload shape, with the windows filled first (the
    window length of untimed steps unless nwarm says otherwise), then nsteps
    timed steps: once as the step runs (mac_decode_step, one launch where it
    applies; events around each step) and once with the match and attention
    kernels launched and timed apart.  K/V values do not change the work of a
    step, so the cache is drawn on the device (seeded N(0, 1), bf16) in the
    workload's layout instead of on the host."""
    import torch
    import kv_cache_reuse_b200 as mac
    nwarm = wl.W if nwarm is None else nwarm
    T = nwarm + nsteps
    stream = synth.queries(wl, T)
    bt_h, max_seq, P = synth.kv_layout(wl, T)
    shape = (wl.B, max_seq, wl.Hkv, wl.D) if bt_h is None else (P, wl.page_size, wl.Hkv, wl.D)
    gen = torch.Generator(device=dev)
    gen.manual_seed(wl.seed)
    K = torch.randn(shape, generator=gen, device=dev, dtype=torch.float32).to(torch.bfloat16).view(torch.int16)
    V = torch.randn(shape, generator=gen, device=dev, dtype=torch.float32).to(torch.bfloat16).view(torch.int16)
    bt = None if bt_h is None else torch.from_numpy(bt_h).to(dev)
    kw = dict(capacity=max_seq) if bt_h is None else dict(max_pages_per_seq=bt_h.shape[1], num_pages=P)
    B, Hq, Hkv, D = wl.B, wl.Hq, wl.Hkv, wl.D
    q = torch.from_numpy(stream.q).to(dev)
    pos = torch.from_numpy(stream.rope_pos).to(dev)
    lens = torch.from_numpy(stream.seq_lens).to(dev)
    out = torch.empty((B, Hq, D), dtype=torch.float32, device=dev)
    lse = torch.empty((B, Hq), dtype=torch.float32, device=dev)
    hit = torch.zeros((T, B, Hkv), dtype=torch.uint8, device=dev)
    mpos = torch.zeros((T, B, Hkv), dtype=torch.int32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    s = torch.cuda.current_stream(dev)
    btp = bt.data_ptr() if bt is not None else None

    def one_pass(split):
        st = mac.MacState.for_workload(wl, **kw)
        for t in range(nwarm):
            st.decode_step(q[t], pos[t], K, V, bt, lens[t], out, lse, hit[t], mpos[t])
            flush.zero_()
        torch.cuda.synchronize(dev)
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(nsteps)]
        h, sp = st.handle, s.cuda_stream
        torch.cuda._sleep(int(2e6 + 4e5 * nsteps))
        for i in range(nsteps):
            t = nwarm + i
            ev[i][0].record(s)
            if split:
                mac.mac_match(h, q[t].data_ptr(), pos[t].data_ptr(), btp, lens[t].data_ptr(), out.data_ptr(),
                              lse.data_ptr(), hit[t].data_ptr(), mpos[t].data_ptr(), sp)
                ev[i][1].record(s)
                mac.mac_attend(h, K.data_ptr(), V.data_ptr(), btp, out.data_ptr(), lse.data_ptr(), sp)
            else:
                mac.mac_decode_step(h, q[t].data_ptr(), pos[t].data_ptr(), K.data_ptr(), V.data_ptr(), btp,
                                    lens[t].data_ptr(), out.data_ptr(), lse.data_ptr(), hit[t].data_ptr(),
                                    mpos[t].data_ptr(), sp)
                ev[i][1].record(s)
            ev[i][2].record(s)
            flush.zero_()
        torch.cuda.synchronize(dev)
        one = mac.mac_one_launch(st)
        status = st.get_status()
        st.close()
        hits = hit.cpu().numpy()[nwarm:]
        mps = mpos.cpu().numpy()[nwarm:]
        mt = at = 0
        for i in range(nsteps):
            a, b_, _ = step_bytes(wl, hits[i], mps[i], stream.seq_lens[nwarm + i], min(nwarm + i, wl.W))
            mt, at = mt + a, at + b_
        m_ms = float(sum(e[0].elapsed_time(e[1]) for e in ev))
        a_ms = float(sum(e[1].elapsed_time(e[2]) for e in ev))
        step_ms = float(sum(e[0].elapsed_time(e[2]) for e in ev))
        return dict(mt=mt, at=at, m_ms=m_ms, a_ms=a_ms, step_ms=step_ms, one=one, status=status,
                    hit_frac=float(hits.mean()))

    r1, r2 = one_pass(False), one_pass(True)
    frac = lambda nbytes, ms: nbytes / (ms * 1e-3) / 1e9 / peak
    return {"workload": wl.name, "batch": B, "q_heads": Hq, "kv_heads": Hkv, "window": wl.W, "band": wl.band,
            "paged": bt_h is not None, "steps": nsteps, "hit_fraction": r1["hit_frac"],
            "step": {"kernel": "mac_step_kernel" if r1["one"] else "mac_match_kernel + mac_attend_kernel",
                     "us": r1["step_ms"] * 1e3 / nsteps, "mb": (r1["mt"] + r1["at"]) / nsteps / 1e6,
                     "frac": frac(r1["mt"] + r1["at"], r1["step_ms"])},
            "attend": {"mb_per_launch": r2["at"] / nsteps / 1e6, "us_per_launch": r2["a_ms"] * 1e3 / nsteps,
                       "achieved": r2["at"] / (r2["a_ms"] * 1e-3) / 1e9, "frac": frac(r2["at"], r2["a_ms"])},
            "match": {"mb_per_launch": r2["mt"] / nsteps / 1e6, "us_per_launch": r2["m_ms"] * 1e3 / nsteps,
                      "achieved": r2["mt"] / (r2["m_ms"] * 1e-3) / 1e9, "frac": frac(r2["mt"], r2["m_ms"])},
            "two_launch_step_us": r2["step_ms"] * 1e3 / nsteps,
            "device_status": max(r1["status"], r2["status"])}


TRACE_PHASES = ("start", "loaded", "decided", "matched", "published", "first_box", "boxes_done", "whole_done",
                "table_built", "table_seen", "range_done", "end")


def run_trace(wl, nsteps, dev, peak):
    """Where the time of a step goes: steps of a workload shape (every labelled
    step a repeat when the workload's stream says so) with the device trace on
    (mac_set_trace), windows filled first.  Per step, each phase's time is
    taken from the first CTA's start, for the median CTA and the last CTA to
    pass it; reported as the median over the steps (microseconds)."""
    import torch
    import kv_cache_reuse_b200 as mac
    nwarm = wl.W
    T = nwarm + nsteps
    stream = synth.queries(wl, T)
    bt_h, max_seq, P = synth.kv_layout(wl, T)
    shape = (wl.B, max_seq, wl.Hkv, wl.D) if bt_h is None else (P, wl.page_size, wl.Hkv, wl.D)
    gen = torch.Generator(device=dev)
    gen.manual_seed(wl.seed)
    K = torch.randn(shape, generator=gen, device=dev, dtype=torch.float32).to(torch.bfloat16).view(torch.int16)
    V = torch.randn(shape, generator=gen, device=dev, dtype=torch.float32).to(torch.bfloat16).view(torch.int16)
    bt = None if bt_h is None else torch.from_numpy(bt_h).to(dev)
    kw = dict(capacity=max_seq) if bt_h is None else dict(max_pages_per_seq=bt_h.shape[1], num_pages=P)
    B, Hq, Hkv, D = wl.B, wl.Hq, wl.Hkv, wl.D
    q = torch.from_numpy(stream.q).to(dev)
    pos = torch.from_numpy(stream.rope_pos).to(dev)
    lens = torch.from_numpy(stream.seq_lens).to(dev)
    out = torch.empty((B, Hq, D), dtype=torch.float32, device=dev)
    lse = torch.empty((B, Hq), dtype=torch.float32, device=dev)
    hit = torch.zeros((B, Hkv), dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    st = mac.MacState.for_workload(wl, **kw)
    mac.mac_set_trace(st, 1)
    med, last, keys = [], [], []
    for t in range(T):
        flush.zero_()
        st.decode_step(q[t], pos[t], K, V, bt, lens[t], out, lse, hit)
        stamps, counters = mac.mac_get_trace(st)
        if t < nwarm:
            continue
        s_ = stamps.astype(np.float64)
        t0 = s_[:, 0][s_[:, 0] > 0].min()
        rel = np.where(s_ > 0, (s_ - t0) * 1e-3, np.nan)
        with np.errstate(all="ignore"):
            med.append(np.nanmedian(rel, axis=0))
            last.append(np.nanmax(rel, axis=0))
        keys.append(int(counters[0]))
    one = mac.mac_one_launch(st)
    st.close()
    with np.errstate(all="ignore"):
        m, l_ = np.nanmedian(np.array(med), axis=0), np.nanmedian(np.array(last), axis=0)
    clean = lambda x: None if not np.isfinite(x) else round(float(x), 2)
    return {"workload": wl.name, "kernel": "mac_step_kernel" if one else "mac_match_kernel + mac_attend_kernel",
            "steps": nsteps, "keys_per_step": float(np.median(keys)),
            "median_cta_us": {n: clean(x) for n, x in zip(TRACE_PHASES, m)},
            "last_cta_us": {n: clean(x) for n, x in zip(TRACE_PHASES, l_)},
            "note": "times from the first CTA's start (%globaltimer), median over steps"}


def run_quality(args, wl, stream, K, V, bt, kw, dev, identity_rope=False):
    """Approximation error of MAC against dense attention on the same stream
    (untimed): one state with the workload's threshold, one with threshold 0
    (every step a miss: dense attention), step by step; per query head the
    relative L2 error of out and the lse difference.  identity_rope rotates
    every query by angle 0 (position 0), which isolates the error of reusing
    a state computed with a query rotated to another position."""
    import torch
    import kv_cache_reuse_b200 as mac
    B, Hq, Hkv, D = wl.B, wl.Hq, wl.Hkv, wl.D
    T = min(args.warmup + args.steps, stream.q.shape[0])
    sm_, sd = mac.MacState.for_workload(wl, **kw), mac.MacState.for_workload(wl, tau=0.0, **kw)
    q = torch.from_numpy(stream.q[:T]).to(dev)
    pos = torch.from_numpy(np.zeros_like(stream.rope_pos[:T]) if identity_rope else stream.rope_pos[:T]).to(dev)
    lens = torch.from_numpy(stream.seq_lens[:T]).to(dev)
    om, od = torch.empty((B, Hq, D), device=dev), torch.empty((B, Hq, D), device=dev)
    lm, ld = torch.empty((B, Hq), device=dev), torch.empty((B, Hq), device=dev)
    hit = torch.empty((B, Hkv), dtype=torch.uint8, device=dev)
    rel_all, rel_hit, dl_hit = [], [], []
    for t in range(T):
        mac.mac_decode_step(sm_, q[t], pos[t], K, V, bt, lens[t], om, lm, hit, None)
        mac.mac_decode_step(sd, q[t], pos[t], K, V, bt, lens[t], od, ld, None, None)
        if t < args.warmup:
            continue
        rel = (torch.linalg.vector_norm(om - od, dim=-1) / torch.linalg.vector_norm(od, dim=-1)).cpu().numpy()
        dl = (lm - ld).abs().cpu().numpy()
        hh = np.repeat(hit.cpu().numpy().astype(bool), Hq // Hkv, axis=1)  # [B][Hq]
        rel_all.append(rel.ravel())
        rel_hit.append(rel[hh])
        dl_hit.append(dl[hh])
    torch.cuda.synchronize(dev)
    status = (sm_.get_status(), sd.get_status())
    sm_.close()
    sd.close()
    ra, rh, dh = np.concatenate(rel_all), np.concatenate(rel_hit), np.concatenate(dl_hit)
    return {"steps": T - args.warmup, "heads_on_hits": int(rh.size),
            "rel_l2_out_mean": float(ra.mean()), "rel_l2_out_on_hits_mean": float(rh.mean()) if rh.size else None,
            "rel_l2_out_on_hits_p99": float(np.percentile(rh, 99)) if rh.size else None,
            "rel_l2_out_on_hits_max": float(rh.max()) if rh.size else None,
            "lse_abs_diff_on_hits_max": float(dh.max()) if dh.size else None,
            "reference": "the same kernels with threshold 0 (dense attention, parity-tested against the fp64 oracle)",
            "device_status": status}


def run_layers(args, wl, stream, cache, K, V, bt, kw, dev, peak):
    """A stack of L independent layers per token -- each with its own state,
    its own copy of the cache and its own query stream -- recorded once as
    one CUDA graph over all layers and replayed per token (the inputs are
    copied into the graph's fixed buffers first, inside the timed region;
    L2 flushed between tokens)."""
    import torch
    import kv_cache_reuse_b200 as mac
    L = args.layers
    B, Hq, Hkv, D = wl.B, wl.Hq, wl.Hkv, wl.D
    T = min(args.warmup + args.steps, stream.q.shape[0])
    s = torch.cuda.current_stream(dev)
    Ks = [K] + [K.clone() for _ in range(L - 1)]
    Vs = [V] + [V.clone() for _ in range(L - 1)]
    q_host = [stream.q[:T]] + [synth.queries(wl.with_(seed=wl.seed + 7919 * l), T).q for l in range(1, L)]
    q_all = torch.from_numpy(np.ascontiguousarray(np.stack(q_host, axis=1))).to(dev)  # [T][L][B][Hq][D]
    pos_all = torch.from_numpy(stream.rope_pos[:T]).to(dev)
    lens_all = torch.from_numpy(stream.seq_lens[:T]).to(dev)
    qb = torch.empty((L, B, Hq, D), dtype=torch.float32, device=dev)
    posb = torch.empty(B, dtype=torch.int32, device=dev)
    lensb = torch.empty(B, dtype=torch.int32, device=dev)
    outs = torch.empty((L, B, Hq, D), dtype=torch.float32, device=dev)
    lses = torch.empty((L, B, Hq), dtype=torch.float32, device=dev)
    hitb = torch.zeros((L, B, Hkv), dtype=torch.uint8, device=dev)
    mpb = torch.zeros((L, B, Hkv), dtype=torch.int32, device=dev)
    hit_all = torch.zeros((T, L, B, Hkv), dtype=torch.uint8, device=dev)
    mp_all = torch.zeros((T, L, B, Hkv), dtype=torch.int32, device=dev)
    states = [mac.MacState.for_workload(wl, **kw) for _ in range(L)]
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    cs = torch.cuda.Stream(dev)
    cs.wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=cs):
        for l in range(L):
            mac.mac_decode_step(states[l], qb[l], posb, Ks[l], Vs[l], bt, lensb, outs[l], lses[l], hitb[l], mpb[l])
    torch.cuda.synchronize(dev)
    ev = []
    for t in range(T):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s)
        qb.copy_(q_all[t])
        posb.copy_(pos_all[t])
        lensb.copy_(lens_all[t])
        g.replay()
        e1.record(s)
        hit_all[t].copy_(hitb)
        mp_all[t].copy_(mpb)
        if t >= args.warmup:
            ev.append((e0, e1))
    torch.cuda.synchronize(dev)
    ms = float(np.sum([a.elapsed_time(b) for a, b in ev]))
    n = len(ev)
    hits = hit_all.cpu().numpy()
    mps = mp_all.cpu().numpy()
    kv = 0
    for t in range(args.warmup, T):
        for l in range(L):
            kv += step_bytes(wl, hits[t, l], mps[t, l], stream.seq_lens[t], min(t, wl.W))[2]
    status = [st.get_status() for st in states]
    for st in states:
        st.close()
    del g
    return {"layers": L, "tokens": n, "tokens_per_s": n / (ms * 1e-3), "ms_per_token": ms / n,
            "us_per_layer": ms * 1e3 / (n * L), "hit_fraction": float(hits[args.warmup:].mean()),
            "kv_bytes_per_token": kv / n, "kv_gbs": kv / (ms * 1e-3) / 1e9, "kv_frac": kv / (ms * 1e-3) / 1e9 / peak,
            "device_status": max(status),
            "timing": "CUDA events around input copies + one graph replay per token; L2 flushed between tokens"}


def run_e2e(args, wl, stream, cache, K, V, bt, kw, dev, world):
    """Same steps through mac_decode_step_host: pinned host inputs (query, positions,
    the step's own K/V rows) copied in, out/lse/hit/match read back, every step."""
    import torch
    import kv_cache_reuse_b200 as mac
    B, Hq, Hkv, D = wl.B, wl.Hq, wl.Hkv, wl.D
    st = mac.MacState.for_workload(wl, **kw)
    s = torch.cuda.current_stream(dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    T = args.warmup + args.steps
    q_h = [torch.from_numpy(stream.q[t]).pin_memory() for t in range(T)]
    p_h = [torch.from_numpy(stream.rope_pos[t]).pin_memory() for t in range(T)]
    l_h = [torch.from_numpy(stream.seq_lens[t]).pin_memory() for t in range(T)]
    rows = [synth.step_rows(cache, stream.seq_lens[t]) for t in range(T)]
    k_h = [torch.from_numpy(r[0].view(np.int16)).pin_memory() for r in rows]
    v_h = [torch.from_numpy(r[1].view(np.int16)).pin_memory() for r in rows]
    out_h = torch.empty((B, Hq, D), dtype=torch.float32).pin_memory()
    lse_h = torch.empty((B, Hq), dtype=torch.float32).pin_memory()
    hit_h = torch.empty((B, Hkv), dtype=torch.uint8).pin_memory()
    mp_h = torch.empty((B, Hkv), dtype=torch.int32).pin_memory()
    tot = 0.0
    for t in range(T):
        flush.zero_()
        torch.cuda.synchronize(dev)
        t0 = time.perf_counter()
        rc = mac.mac_decode_step_host(st, q_h[t], p_h[t], l_h[t], k_h[t], v_h[t], K, V, bt, out_h, lse_h, hit_h,
                                      mp_h, s)
        t1 = time.perf_counter()
        if rc != mac.MAC_OK:
            raise RuntimeError("device status %d in e2e step" % mac.mac_get_status(st))
        if t >= args.warmup:
            tot += t1 - t0
    st.close()
    tot = max_over_ranks(tot, world, dev)
    # one packed block each way, fields padded to 256 bytes (the status word rides in the output block)
    up = lambda x: (x + 255) // 256 * 256
    h2d = up(B * Hq * D * 4) + up(B * 4) + up(B * 4) + up(B * Hkv * D * 2) + up(B * Hkv * D * 2)
    d2h = up(B * Hq * D * 4) + up(B * Hq * 4) + up(B * Hkv) + up(B * Hkv * 4) + 16
    return {"value": world * args.steps / tot, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "timer": "host wall clock around each mac_decode_step_host call (it synchronises)"}


def run_cpu_baseline(wl, stream, cache, seconds):
    """The fp64 oracle on the host cores, on the first steps of the same stream
    (bounded to about `seconds` of CPU work): steps/s overall and split by
    step kind (every unit hit / some unit missed), and GB/s of bf16 K/V read."""
    import oracle
    orc = oracle.Oracle.for_workload(wl, cache)
    t0 = time.perf_counter()
    n = nh = 0
    kv = 0
    kind_s = {"all_hit": [0, 0.0], "with_miss": [0, 0.0]}
    while n < stream.q.shape[0]:
        ts = time.perf_counter()
        r = orc.step(stream.q[n], stream.rope_pos[n], cache.K, cache.V, cache.block_table, stream.seq_lens[n])
        te = time.perf_counter()
        nh += int(r.hit.sum())
        kv += int(r.keys_read) * 2 * wl.D * 2  # K and V rows of every key a unit read
        k = kind_s["all_hit" if r.hit.all() else "with_miss"]
        k[0] += 1
        k[1] += te - ts
        n += 1
        if te - t0 > seconds:
            break
    dt = time.perf_counter() - t0
    return {"value": n / dt, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
            "kv_gbs": kv / dt / 1e9,
            "steps_per_s_by_kind": {k: (v[0] / v[1] if v[1] > 0 else None) for k, v in kind_s.items()},
            "steps_by_kind": {k: v[0] for k, v in kind_s.items()},
            "sample": "first %d decode steps of %s from an empty window (%d of %d unit decisions hit), %.1f s" % (
                n, wl.name, nh, n * wl.B * wl.Hkv, dt)}


def run_reference(args, rank, world):
    """--impl reference: the fp64 CPU oracle as it stands, on the host cores."""
    if rank != 0:
        return None
    import oracle
    wl = synth.WORKLOADS[args.workload]
    T = max(wl.steps, args.warmup + args.steps)
    stream = synth.queries(wl, T)
    cache = synth.kv_cache(wl, T)
    orc = oracle.Oracle.for_workload(wl, cache)
    for t in range(args.warmup):
        orc.step(stream.q[t], stream.rope_pos[t], cache.K, cache.V, cache.block_table, stream.seq_lens[t])
    t0 = time.perf_counter()
    n = 0
    for t in range(args.warmup, args.warmup + args.steps):
        orc.step(stream.q[t], stream.rope_pos[t], cache.K, cache.V, cache.block_table, stream.seq_lens[t])
        n += 1
        if time.perf_counter() - t0 > args.cpu_seconds * 6:
            break
    dt = time.perf_counter() - t0
    v = n / dt
    sample = "decode steps %d..%d of %s (fp64 oracle, every unit of every step)" % (args.warmup, args.warmup + n - 1,
                                                                                    wl.name)
    return {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": world, "steps": n,
            "warmup": args.warmup, "ms_per_step": 1e3 * dt / n, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": bench_config(wl, cache.paged, world),
            "cpu_baseline": {"value": v, "unit": UNIT, "kind": "oracle", "cores": oracle.num_threads(),
                             "sample": sample},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=120)
    ap.add_argument("--warmup", type=int, default=8)
    ap.add_argument("--impl", default="mac", choices=["mac", "reference"])
    ap.add_argument("--workload", default="long_128k", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--miss-steps", type=int, default=16, help="timed steps of the all-miss run (0 = skip)")
    ap.add_argument("--hit-steps", type=int, default=16, help="timed steps of the all-hit run (0 = skip)")
    ap.add_argument("--warm-start", action="store_true", help="also time seeding the windows from W positions")
    ap.add_argument("--layers", type=int, default=4,
                    help="also time a stack of this many layers per token, one CUDA graph per token (0 = skip)")
    ap.add_argument("--trace-steps", type=int, default=12,
                    help="steps of the device phase trace runs (0 = skip)")
    ap.add_argument("--no-paged-gap", dest="paged_gap", action="store_false",
                    help="skip the paged-against-contiguous all-miss runs")
    ap.add_argument("--mqa-steps", type=int, default=8,
                    help="timed steps of the 32-query-heads-over-one-KV-head runs (0 = skip)")
    ap.add_argument("--hit-shapes", default="paged_mixed,continuous_16k",
                    help="workloads whose shapes also get an all-hit run (comma-separated, empty = none)")
    ap.add_argument("--no-bf16", action="store_true", help="skip the bf16 query / window run")
    ap.add_argument("--no-per-head", action="store_true", help="skip the per-head matching run")
    ap.add_argument("--no-quality", action="store_true", help="skip the approximation-error pass")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=20.0)
    ap.add_argument("--batch", type=int, default=0, help="override the workload's batch (profiling of smaller cases)")
    ap.add_argument("--tau", type=float, default=None, help="override the match threshold (0 = every step misses)")
    ap.add_argument("--q-heads", type=int, default=0, help="override the query heads (other group sizes)")
    ap.add_argument("--kv-heads", type=int, default=0, help="override the KV heads (other group sizes)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        res = run_reference(args, rank, world)
    else:
        if world > 1:
            import datetime
            import torch
            torch.cuda.set_device(local_rank)
            torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=600))
        res = run_mac(args, rank, world, local_rank)
        if world > 1:
            import torch
            torch.distributed.barrier()
            torch.distributed.destroy_process_group()
    if res is not None:
        if isinstance(res, tuple):
            res, detail = res
            print(json.dumps(dict(detail, metric=res["metric"], value=res["value"])), file=sys.stderr, flush=True)
        print(json.dumps(_compact(res)), flush=True)


def _compact(x, digits=5):
    """The result with every float rounded to `digits` significant digits
    (keeps the one JSON line short; the full-precision record is on stderr)."""
    if isinstance(x, float):
        return float("%.*g" % (digits, x)) if math.isfinite(x) else x
    if isinstance(x, dict):
        return {k: _compact(v, digits) for k, v in x.items()}
    if isinstance(x, (list, tuple)):
        return [_compact(v, digits) for v in x]
    return x


if __name__ == "__main__":
    main()
