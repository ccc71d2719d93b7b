"""Benchmark of the Star / Pulsar two-phase attention hot path on B200.

One step = one pass of the whole path over one 128K-token sequence of the
Llama-3.1-8B attention shape (32 q / 8 kv heads, d = 128, bf16, RoPE theta
500000, 8 blocks of 16384, 64-token sink, 32-token chunks, 2048-token
summaries): Max-IDF selection -> Pulsar Phase-1 encoding of all 8 hosts ->
Phase-2 attention of a 64-token query over the 8 retained shards with the
exact LSE merge.  value = context tokens encoded per second (whole job).

Also measured in the same run (reported beside the headline, not as bench
lines of their own): the Star anchor-variant Phase 1 on the same input, and
the Phase-2 decode of 16 single-token queries over a 128K bf16 cache in 8
shards (GB/s against HBM).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (torchrun, one process per GPU) the default is the method's own
multi-GPU layout (`--layout hosts`): the 8 hosts of ONE sequence spread over
the ranks in contiguous ranges balanced by attention work (Phase 1 without
communication), then the Phase-2 exchange -- every rank's shard partials
all-gathered over NCCL and merged exactly (strong scaling); the time is the
max over ranks.  `--layout sequences` gives every rank its own independent
sequence instead (weak scaling, no data-path collective); on one GPU the two
are the same work and `sequences` is the default (`--layout hosts` then runs
the exchange in a process group of one rank).  `--impl reference` times the
fp64 CPU oracle on a fixed sample of the same step (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from long_context_blockwise_max_b200 import workloads  # noqa: E402

METRIC = "Phase-1 encode tokens/s (%bf16 TC peak); Phase-2 query attn GB/s (%HBM) @128K"
WORKLOAD = workloads.LLAMA_128K
DECODE = workloads.DECODE_128K
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# NVIDIA's nominal B200 figures, reported beside the measured denominators
NOMINAL_BF16_TFLOPS = 2250.0   # dense
NOMINAL_HBM_GBS = 8000.0


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


TRAFFIC_FILE = os.path.join(ROOT, "profiles", "roofline_traffic.txt")


def source_digest(paths):
    """sha256 over the given source files (repository-relative paths)."""
    import hashlib
    h = hashlib.sha256()
    for rel in paths:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch of `kernel` on `workload` recorded from an ncu
    capture in profiles/roofline_traffic.txt (one record per kernel, each
    starting at its `kernel` line), or None when there is none or the
    kernel's sources changed since it was taken."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    records, rec = [], None
    for line in open(TRAFFIC_FILE):
        line = line.strip()
        if line and not line.startswith("#"):
            key, _, val = line.partition(" ")
            if key == "kernel":
                rec = {}
                records.append(rec)
            if rec is not None:
                rec[key] = val.strip()
    for rec in records:
        if rec.get("kernel") != kernel or rec.get("workload") != workload:
            continue
        try:
            if source_digest(rec["sources"].split()) != rec["sources_sha256"]:
                return None
            return int(rec["dram_bytes_read"]) + int(rec["dram_bytes_write"])
        except (KeyError, OSError, ValueError):
            return None
    return None


# --------------------------------------------------------------------------
# clocks during the timed region
# --------------------------------------------------------------------------
class ClockSampler:
    """nvidia-smi sampling every 50 ms, started well before the timed region
    (the tool takes a few hundred ms to produce its first line) and summarised
    over the samples whose timestamps fall inside the window marked with
    mark_start() / mark_end()."""
    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.t_start = self.t_end = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        import atexit
        atexit.register(self._stop)   # no sampler outlives the run, even after an error
        return self

    def _stop(self):
        if self.proc is not None and self.proc.poll() is None:
            self.proc.kill()

    def mark_start(self):
        self.t_start = time.time()

    def mark_end(self):
        self.t_end = time.time()

    def __exit__(self, *exc):
        self.out = ""
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()
        return False

    @staticmethod
    def _epoch(stamp: str):
        import datetime
        try:
            return datetime.datetime.strptime(stamp, "%Y/%m/%d %H:%M:%S.%f").timestamp()
        except ValueError:
            return None

    def summary(self):
        """Median SM clock, maximum clock and the throttle reasons seen over
        the samples inside the marked window (all samples if the window holds
        none, with "in_window": false)."""
        rows = []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in (self.out or "").strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                rows.append((self._epoch(f[0]), float(f[1]), float(f[2]),
                             {n for n, val in zip(names, f[5:9]) if val.lower().startswith("active")}))
            except ValueError:
                continue
        inside = [r for r in rows if r[0] is not None and self.t_start is not None and self.t_end is not None
                  and self.t_start <= r[0] <= self.t_end]
        use = inside or rows
        if not use:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(r[1] for r in use), "sm_max_mhz": max(r[2] for r in use),
                "reasons": sorted(set().union(*(r[3] for r in use))), "samples": len(use),
                "in_window": bool(inside)}


# --------------------------------------------------------------------------
# our implementation
# --------------------------------------------------------------------------
class Step:
    """Preallocated buffers and the calls of one hot-path step.

    ``hosts = (h0, h1, group, max_local)`` runs the multi-GPU layout of the
    method on this rank: Phase 1 of hosts [h0, h1) of the sequence, then the
    Phase-2 exchange (the rank's shard partials, an NCCL all-gather over
    ``group`` with every rank padded to ``max_local`` shards, the exact
    merge)."""

    def __init__(self, w, dev, seed_offset=0, hosts=None):
        from long_context_blockwise_max_b200 import pulsar as P
        self.P, self.w, self.dev = P, w, dev
        self.hosts = hosts
        ids = w.token_ids()
        if seed_offset:
            ids = np.roll(ids, seed_offset * 4099)
        self.ids_h = torch.from_numpy(ids).pin_memory() if torch.cuda.is_available() else torch.from_numpy(ids)
        q, k, v = w.qkv(device=dev)
        self.q, self.k, self.v = q, k, v
        self.query = w.query(device=dev)
        self.ids = self.ids_h.to(dev)
        n = w.n_blocks
        summ = w.k_chunks * w.chunk
        self.row_off = P.pa_phase1_layout(w.L, w.block, w.sink, summ, False)
        h0, h1 = (hosts[0], hosts[1]) if hosts else (0, n)
        self.h0, self.h1 = h0, h1
        R = self.row_off[h1] - self.row_off[h0]
        self.sel = torch.empty((n, w.k_chunks), dtype=torch.int32, device=dev)
        self.ws_sel = torch.empty(P.pa_select_workspace_size(w.L, w.vocab, w.block, w.chunk), dtype=torch.uint8,
                                  device=dev)
        self.o1 = torch.empty((max(R, 1), w.hq, w.d), dtype=w.dtype, device=dev)
        self.lse1 = torch.empty((max(R, 1), w.hq), dtype=torch.float32, device=dev)
        nret = (h1 - h0) * w.block
        self.k_ret = torch.empty((max(nret, 1), w.hkv, w.d), dtype=w.dtype, device=dev)
        self.v_ret = torch.empty_like(self.k_ret)
        self.ws1 = torch.empty(max(P.pa_phase1_hosts_workspace_size(w.L, w.hq, w.hkv, w.d, 1, w.block, w.sink, summ,
                                                                    False, h0, h1), 256),
                               dtype=torch.uint8, device=dev)
        self.o2 = torch.empty_like(self.query)
        self.lse2 = torch.empty((1, w.q_tokens, w.hq), dtype=torch.float32, device=dev)
        self.ws2 = torch.empty(P.pa_phase2_workspace_size(1, w.q_tokens, max(nret, 1), max(h1 - h0, 1), w.hq, w.hkv,
                                                          w.d), dtype=torch.uint8, device=dev)
        if hosts:
            self.part_o = torch.empty((1, max(h1 - h0, 1), w.q_tokens, w.hq, w.d), dtype=torch.float32, device=dev)
            self.part_lse = torch.empty((1, max(h1 - h0, 1), w.q_tokens, w.hq), dtype=torch.float32, device=dev)
        self.attn_events = None
        self.p2_events = None
        self.stage_events = None   # 4 events: before selection, after it, after Phase 1, after Phase 2

    def run(self):
        P, w = self.P, self.w
        ev = self.stage_events
        if ev:
            ev[0].record()
        P.pulsar_select_summaries(self.ids, w.vocab, w.block, w.chunk, w.k_chunks, sel=self.sel, ws=self.ws_sel)
        if ev:
            ev[1].record()
        P.pa_set_profile_events(*(self.attn_events or (None, None)))
        if self.hosts:
            P.pulsar_phase1_encode_hosts(self.q, self.k, self.v, w.rope_theta, w.block, w.sink, w.chunk,
                                         w.k_chunks, self.sel, self.h0, self.h1, o=self.o1, lse=self.lse1,
                                         k_ret=self.k_ret, v_ret=self.v_ret, ws=self.ws1)
        else:
            P.pulsar_phase1_encode(self.q, self.k, self.v, w.rope_theta, w.block, w.sink, w.chunk, w.k_chunks,
                                   self.sel, o=self.o1, lse=self.lse1, k_ret=self.k_ret, v_ret=self.v_ret,
                                   ws=self.ws1)
        if ev:
            ev[2].record()
        P.pa_set_profile_events(*(self.p2_events or (None, None)))
        if self.hosts:
            self._exchange()
        else:
            P.star_phase2_attend(self.query, self.k_ret[None], self.v_ret[None], w.n_blocks, q_pos0=w.L,
                                 rope_theta=w.rope_theta, o=self.o2, lse=self.lse2, ws=self.ws2)
        P.pa_set_profile_events(None, None)
        if ev:
            ev[3].record()

    def _exchange(self):
        """Phase 2 of the multi-GPU layout: this rank's shards' partials, the
        NCCL all-gather of every rank's partials, the exact merge."""
        from long_context_blockwise_max_b200 import distributed as D
        P, w = self.P, self.w
        n_local = self.h1 - self.h0

        def partials(q, kl, vl, n, q_pos0, theta):
            P.star_phase2_attend(q, kl, vl, n, q_pos0=q_pos0, rope_theta=theta, o=self.o2, lse=self.lse2,
                                 want_partials=True, part_o=self.part_o, part_lse=self.part_lse, ws=self.ws2)
            return self.part_o, self.part_lse

        def merge(all_o, all_lse, dtype):
            return P.pa_lse_merge(all_o, all_lse, dtype=dtype, o=self.o2, lse=self.lse2)
        nret = n_local * w.block
        D.phase2_attend_distributed(self.query, self.k_ret[None, :nret], self.v_ret[None, :nret], n_local,
                                    w.n_blocks, w.L, w.rope_theta, group=self.hosts[2], partials_fn=partials,
                                    merge_fn=merge, max_local=self.hosts[3])

    def launches(self):
        """Kernels of ours one step launches (bf16, as in the ncu launch list
        of the step): selection 3 (presence, min df, top-k); Phase 1 4 (row
        map, RoPE, attention, the fp32 pass over each host's first rows) plus
        the position map of a compact host range; Phase 2 4 (query RoPE,
        tensor-core partials, the exact pass over units with keys beyond fp16
        range, merge) plus the exchange's merge of the gathered partials."""
        n = 11
        if self.hosts:
            w, h0, h1 = self.w, self.h0, self.h1
            pre = w.sink + (h1 - 1) * w.k_chunks * w.chunk
            n += 1 + (1 if h1 >= 2 and pre + (h1 - h0) * w.block < h1 * w.block else 0)
        return n

    def check_status(self, where):
        """Device status of the step's three workspaces (selection, Phase 1,
        Phase 2); a run whose kernels reported an error yields no number."""
        for name, ws in (("selection", self.ws_sel), ("Phase 1", self.ws1), ("Phase 2", self.ws2)):
            st = self.P.pa_workspace_status(ws)
            if st != 0:
                raise RuntimeError(f"{name} device status {st} ({self.P.status_string(st)}) {where}")


def require_ok(P, ws, what):
    """Raise if a side measurement's kernels reported a device error."""
    st = P.pa_workspace_status(ws)
    if st != 0:
        raise RuntimeError(f"{what}: device status {st} ({P.status_string(st)})")


def host_lengths(w, star):
    n = w.n_blocks
    summ = w.k_chunks * w.chunk
    return [w.block] + [(2 * w.block if star else w.sink + i * summ + w.block) for i in range(1, n)]


def attn_flops(w, star=False, hosts=None):
    """Algorithmic Phase-1 FLOPs: 4 * d * Hq * n(n+1)/2 per host (QK^T and PV
    over the causal pairs, diagonal included; softmax not counted), over all
    hosts or hosts [h0, h1)."""
    ns = host_lengths(w, star)
    if hosts is not None:
        ns = ns[hosts[0]:hosts[1]]
    return float(sum(4.0 * w.d * w.hq * n * (n + 1) / 2.0 for n in ns))


def sync_all(dist_on, device="cuda"):
    """Barrier across ranks with the device drained on both sides."""
    if str(device).startswith("cuda"):
        torch.cuda.synchronize()
    if dist_on:
        torch.distributed.barrier()
        if str(device).startswith("cuda"):
            torch.cuda.synchronize()


def max_over_ranks(x: float, dist_on: bool, device="cuda") -> float:
    """The largest of the ranks' values (every rank gets it)."""
    if not dist_on:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: float, world: int, ms_per_step: float) -> float:
    """Units processed by all ranks per second, timed by the slowest rank."""
    return units_per_rank * world / (ms_per_step * 1e-3)


def run_ours(args, rank, world, local_rank, dist_on):
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    clk = ClockSampler(local_rank).__enter__()   # running before the timed region starts
    w = WORKLOAD
    peaks, peak_kind = load_peaks()
    hosts_layout = args.layout == "hosts"
    if hosts_layout:
        # one sequence, its hosts spread over the ranks (Phase 1 without
        # communication, then the Phase-2 all-gather over NCCL)
        from long_context_blockwise_max_b200.distributed import phase1_host_ranges
        ranges = phase1_host_ranges(w.L, w.block, w.sink, w.chunk, w.k_chunks, False, world)
        h0, h1 = ranges[rank]
        step = Step(w, dev, hosts=(h0, h1, torch.distributed.group.WORLD, max(b - a for a, b in ranges)))
    else:
        h0, h1 = 0, w.n_blocks
        step = Step(w, dev, seed_offset=rank)
    for _ in range(args.warmup):
        step.run()
    step.check_status("after warm-up")

    # ---- timed region: K steps -----------------------------------------
    K = args.steps
    ev_attn = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    ev_p2 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    ev_stage = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(4)) for _ in range(K)]
    for a, b in ev_attn + ev_p2:      # torch creates the CUDA event on its first record
        a.record()
        b.record()
    for evs in ev_stage:
        for e in evs:
            e.record()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sync_all(dist_on)
    clk.mark_start()
    t0.record()
    for i in range(K):
        step.attn_events = ev_attn[i]
        step.p2_events = ev_p2[i]
        step.stage_events = ev_stage[i]
        step.run()
    t1.record()
    torch.cuda.synchronize()
    clk.mark_end()
    clk.__exit__(None, None, None)
    step.attn_events = None
    step.p2_events = None
    step.stage_events = None
    sync_all(dist_on)
    step.check_status("after the timed steps")
    ms = max_over_ranks(t0.elapsed_time(t1), dist_on) / K
    # a rank with no host (more ranks than hosts) launches no attention kernel
    attn_ms = statistics.mean(a.elapsed_time(b) for a, b in ev_attn) if h1 > h0 else float("nan")
    p2_ms = statistics.mean(a.elapsed_time(b) for a, b in ev_p2)
    sel_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in ev_stage)
    enc_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in ev_stage)
    p2_call_ms = statistics.mean(e[2].elapsed_time(e[3]) for e in ev_stage)

    flops = attn_flops(w, hosts=(h0, h1))
    # whole job: one sequence per rank, or one sequence spread over the ranks
    tokens_per_s = w.L / (ms * 1e-3) if hosts_layout else whole_job_rate(w.L, world, ms)
    # the burst peak: the timed region is a fraction of a second, not the
    # seconds-long loop the sustained figure was measured over
    peak_tf = peaks["bf16_tflops"]
    attn_tf = flops / (attn_ms * 1e-3) / 1e12

    # ---- end to end through the public API with host buffers ------------
    # Every step copies its inputs from pinned host memory and reads its
    # Phase-2 result back.  Two sets of device input buffers let the copy of
    # step i+1 (copy stream) run under the compute of step i (compute stream).
    q_h = step.q.cpu().pin_memory()
    k_h = step.k.cpu().pin_memory()
    v_h = step.v.cpu().pin_memory()
    query_h = step.query.cpu().pin_memory()
    hosts_in = (step.ids_h, q_h, k_h, v_h, query_h)
    o2_h = [torch.empty(step.o2.shape, dtype=step.o2.dtype).pin_memory() for _ in range(2)]
    lse2_h = [torch.empty(step.lse2.shape, dtype=torch.float32).pin_memory() for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in hosts_in)
    d2h = o2_h[0].numel() * o2_h[0].element_size() + lse2_h[0].numel() * 4
    bufs = [(step.ids, step.q, step.k, step.v, step.query),
            tuple(torch.empty_like(t) for t in (step.ids, step.q, step.k, step.v, step.query))]
    copy_s, comp_s = torch.cuda.Stream(), torch.cuda.Stream()
    copied = [torch.cuda.Event() for _ in range(2)]
    consumed = [torch.cuda.Event() for _ in range(2)]

    def e2e_steps(n):
        for i in range(n):
            b = i % 2
            with torch.cuda.stream(copy_s):
                if i >= 2:
                    copy_s.wait_event(consumed[b])
                for dst, src in zip(bufs[b], hosts_in):
                    dst.copy_(src, non_blocking=True)
                copied[b].record(copy_s)
            with torch.cuda.stream(comp_s):
                comp_s.wait_event(copied[b])
                step.ids, step.q, step.k, step.v, step.query = bufs[b]
                step.run()
                consumed[b].record(comp_s)
                o2_h[b].copy_(step.o2, non_blocking=True)
                lse2_h[b].copy_(step.lse2, non_blocking=True)

    e2e_steps(2)
    torch.cuda.synchronize()
    sync_all(dist_on)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    copy_s.wait_event(e0)
    e2e_steps(K)
    torch.cuda.current_stream().wait_stream(comp_s)
    torch.cuda.current_stream().wait_stream(copy_s)
    e1.record()
    torch.cuda.synchronize()
    sync_all(dist_on)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dist_on) / K
    step.ids, step.q, step.k, step.v, step.query = bufs[0]
    step.check_status("after the end-to-end steps")
    e2e_rate = w.L / (e2e_ms * 1e-3) if hosts_layout else whole_job_rate(w.L, world, e2e_ms)

    # ---- side measurements: Star Phase 1, Phase-2 decode ----------------
    P = step.P
    extra = {}
    if not args.headline_only and not hosts_layout:
        row_star = P.pa_phase1_layout(w.L, w.block, 0, 0, True)[-1]
        o_star = torch.empty((row_star, w.hq, w.d), dtype=w.dtype, device=dev)
        ws_star = torch.empty(P.pa_phase1_workspace_size(w.L, w.hq, w.hkv, w.d, 1, w.block, 0, 0, True),
                              dtype=torch.uint8, device=dev)
        del step.o1, step.lse1
        torch.cuda.empty_cache()

        def star():
            P.star_phase1_encode(step.q, step.k, step.v, w.rope_theta, w.block, o=o_star, lse=None,
                                 k_ret=step.k_ret, v_ret=step.v_ret, ws=ws_star, want_lse=False)
        star()
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = max(1, min(K, 3))
        torch.cuda.synchronize()
        s0.record()
        for _ in range(reps):
            star()
        s1.record()
        torch.cuda.synchronize()
        star_ms = s0.elapsed_time(s1) / reps
        require_ok(P, ws_star, "Star Phase 1")
        sf = attn_flops(w, star=True)
        extra["star_phase1"] = {"ms": round(star_ms, 3), "tflop": round(sf / 1e12, 3),
                                "tflop_s": round(sf / (star_ms * 1e-3) / 1e12, 1),
                                "flop_ratio_star_over_pulsar": round(sf / flops, 3)}
        del o_star, ws_star
        torch.cuda.empty_cache()

        dq, dk, dv = DECODE.decode_inputs(device=dev)
        B, T, S = DECODE.decode_batch, DECODE.decode_T, DECODE.decode_shards
        do = torch.empty_like(dq)
        dl = torch.empty((B, 1, DECODE.hq), dtype=torch.float32, device=dev)
        dws = torch.empty(P.pa_phase2_workspace_size(B, 1, T, S, DECODE.hq, DECODE.hkv, DECODE.d),
                          dtype=torch.uint8, device=dev)
        pev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
        for a, b in pev:
            a.record()
            b.record()

        def dec():
            P.star_phase2_attend(dq, dk, dv, S, q_pos0=T, rope_theta=DECODE.rope_theta, o=do, lse=dl, ws=dws)
        for _ in range(3):
            dec()
        torch.cuda.synchronize()
        d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        d0.record()
        for i in range(K):
            P.pa_set_profile_events(*pev[i])
            dec()
        P.pa_set_profile_events(None, None)
        d1.record()
        torch.cuda.synchronize()
        dec_ms = d0.elapsed_time(d1) / K
        require_ok(P, dws, "128K decode")
        dec_kernel_ms = statistics.mean(a.elapsed_time(b) for a, b in pev)
        kv_bytes = 2.0 * B * T * DECODE.hkv * DECODE.d * 2
        extra["phase2_decode"] = {
            "workload": DECODE.name, "ms": round(dec_ms, 4), "kernel_ms": round(dec_kernel_ms, 4),
            "gb_s": round(kv_bytes / (dec_ms * 1e-3) / 1e9, 1),
            "kernel_gb_s": round(kv_bytes / (dec_kernel_ms * 1e-3) / 1e9, 1),
            "frac_hbm": round(kv_bytes / (dec_ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
            "frac_of_nominal_hbm": round(kv_bytes / (dec_ms * 1e-3) / 1e9 / NOMINAL_HBM_GBS, 4),
            "bytes_per_call": kv_bytes}
        # ART early termination on the same decode (the page's defaults)
        ao = torch.empty_like(dq)
        al = torch.empty((B, 1, DECODE.hq), dtype=torch.float32, device=dev)
        aws = torch.empty(P.pa_phase2_workspace_size(B, 1, T, 1, DECODE.hq, DECODE.hkv, DECODE.d),
                          dtype=torch.uint8, device=dev)

        def art():
            return P.star_phase2_attend_art(dq, dk, dv, T, DECODE.rope_theta, o=ao, lse=al, ws=aws)
        for _ in range(3):
            art()
        torch.cuda.synchronize()
        r0, r1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        r0.record()
        for _ in range(K):
            _, _, vis, _ = art()
        r1.record()
        torch.cuda.synchronize()
        art_ms = r0.elapsed_time(r1) / K
        require_ok(P, aws, "ART decode")
        frac = float(vis.float().mean().item()) * 128 / T
        extra["phase2_decode_art"] = {"ms": round(art_ms, 4), "visited_fraction": round(frac, 4),
                                      "gb_s_of_visited": round(kv_bytes * frac / (art_ms * 1e-3) / 1e9, 1),
                                      "tau": 1e-5, "phi": 1e-3, "patience": 5, "block_keys": 128}
        # ART where its stop applies: the same decode shape with the keys older
        # than the newest 4096 moved by -60 along the normalised sum of their
        # kv group's query vectors (no RoPE), so that their softmax weights
        # are about e^-30 and the output settles once the recent keys are in;
        # timed against the exact decode on the same cache
        W = 4096
        g = DECODE.hq // DECODE.hkv
        u = dq.float().view(B, 1, DECODE.hkv, g, DECODE.d).sum(3)
        u = u / u.norm(dim=-1, keepdim=True)
        dk2 = dk.clone()
        for b0 in range(B):
            dk2[b0, :T - W] = (dk2[b0, :T - W].float() - 60.0 * u[b0]).to(dk.dtype)
        eo = torch.empty_like(dq)
        el = torch.empty((B, 1, DECODE.hq), dtype=torch.float32, device=dev)
        ews = torch.empty(P.pa_phase2_workspace_size(B, 1, T, DECODE.decode_shards, DECODE.hq, DECODE.hkv, DECODE.d),
                          dtype=torch.uint8, device=dev)

        def art2():
            return P.star_phase2_attend_art(dq, dk2, dv, T, 0.0, o=ao, lse=al, ws=aws)

        def exact2():
            P.star_phase2_attend(dq, dk2, dv, DECODE.decode_shards, T, 0.0, o=eo, lse=el, ws=ews)

        def timed(fn):
            for _ in range(3):
                fn()
            torch.cuda.synchronize()
            x0, x1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            x0.record()
            for _ in range(K):
                out = fn()
            x1.record()
            torch.cuda.synchronize()
            return x0.elapsed_time(x1) / K, out
        art2_ms, (_, _, vis2, _) = timed(art2)
        ex2_ms, _ = timed(exact2)
        frac2 = float(vis2.float().mean().item()) * 128 / T
        require_ok(P, aws, "ART decode, recency cache")
        require_ok(P, ews, "exact decode, recency cache")
        extra["phase2_decode_art_recency"] = {
            "ms": round(art2_ms, 4), "exact_ms": round(ex2_ms, 4), "speedup": round(ex2_ms / art2_ms, 2),
            "visited_fraction": round(frac2, 4),
            "max_abs_o_diff_vs_exact": round(float((ao.float() - eo.float()).abs().max().item()), 5),
            "max_abs_lse_diff_vs_exact": round(float((al - el).abs().max().item()), 6),
            "cache": "decode_128k_b16 with keys older than the newest 4096 moved by -60 along the group's "
                     "normalised query sum; no RoPE"}
        del dq, dk, dv, dk2
        torch.cuda.empty_cache()

        # the 1M-token decode: batch 4 over a 16 GiB cache in 32 shards
        SC = workloads.SCALE_1M
        sq, sk, sv = SC.decode_inputs(device=dev)
        B1, T1, S1 = SC.decode_batch, SC.decode_T, SC.decode_shards
        so_ = torch.empty_like(sq)
        sl_ = torch.empty((B1, 1, SC.hq), dtype=torch.float32, device=dev)
        sws = torch.empty(P.pa_phase2_workspace_size(B1, 1, T1, S1, SC.hq, SC.hkv, SC.d), dtype=torch.uint8,
                          device=dev)

        def dec1m():
            P.star_phase2_attend(sq, sk, sv, S1, q_pos0=T1, rope_theta=SC.rope_theta, o=so_, lse=sl_, ws=sws)
        dec1m_ms, _ = timed(dec1m)
        require_ok(P, sws, "1M decode")
        kv1m = 2.0 * B1 * T1 * SC.hkv * SC.d * 2
        extra["phase2_decode_1m"] = {
            "workload": SC.name, "ms": round(dec1m_ms, 4), "gb_s": round(kv1m / (dec1m_ms * 1e-3) / 1e9, 1),
            "frac_hbm": round(kv1m / (dec1m_ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4), "bytes_per_call": kv1m}
        del sq, sk, sv
        torch.cuda.empty_cache()

        # generation loop on the query host: the 64-token query, then 128
        # tokens generated one at a time over the retained 128K cache
        gen = 128
        ng = w.q_tokens + gen
        gq = workloads.normal((1, ng, w.hq, w.d), workloads.SEED_QUERY + 10, w.dtype, dev)
        gk = workloads.normal((1, ng, w.hkv, w.d), workloads.SEED_QUERY + 11, w.dtype, dev)
        gv = workloads.normal((1, ng, w.hkv, w.d), workloads.SEED_QUERY + 12, w.dtype, dev)
        ks = torch.zeros((1, ng, w.hkv, w.d), dtype=w.dtype, device=dev)
        vs = torch.zeros_like(ks)
        kr1, vr1 = step.k_ret[None], step.v_ret[None]
        go = torch.empty((1, 1, w.hq, w.d), dtype=w.dtype, device=dev)
        gl = torch.empty((1, 1, w.hq), dtype=torch.float32, device=dev)
        gws = torch.empty(P.pa_phase2_workspace_size(1, w.q_tokens, w.L, w.n_blocks, w.hq, w.hkv, w.d),
                          dtype=torch.uint8, device=dev)
        P.star_phase2_query_step(gq[:, :w.q_tokens].contiguous(), gk[:, :w.q_tokens].contiguous(),
                                 gv[:, :w.q_tokens].contiguous(), kr1, vr1, w.n_blocks, ks, vs, 0, w.L,
                                 w.rope_theta, ws=gws)
        toks = [(gq[:, t:t + 1].contiguous(), gk[:, t:t + 1].contiguous(), gv[:, t:t + 1].contiguous())
                for t in range(w.q_tokens, ng)]
        torch.cuda.synchronize()
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record()
        for i, (a_q, a_k, a_v) in enumerate(toks):
            t = w.q_tokens + i
            P.star_phase2_query_step(a_q, a_k, a_v, kr1, vr1, w.n_blocks, ks, vs, t, w.L + t, w.rope_theta,
                                     o=go, lse=gl, ws=gws)
        g1.record()
        torch.cuda.synchronize()
        gen_ms = g0.elapsed_time(g1) / gen
        require_ok(P, gws, "generation steps")
        # the same 128 steps captured once in a CUDA graph and replayed (each
        # replay rewrites the same own-cache rows): GPU time per token without
        # the Python / ctypes cost of the per-token call
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for i, (a_q, a_k, a_v) in enumerate(toks):
                t = w.q_tokens + i
                P.star_phase2_query_step(a_q, a_k, a_v, kr1, vr1, w.n_blocks, ks, vs, t, w.L + t, w.rope_theta,
                                         o=go, lse=gl, ws=gws)
        graph.replay()
        torch.cuda.synchronize()
        g0.record()
        graph.replay()
        g1.record()
        torch.cuda.synchronize()
        gen_graph_ms = g0.elapsed_time(g1) / gen
        del graph
        cache_bytes = 2.0 * w.L * w.hkv * w.d * 2
        extra["generation"] = {"context": w.L, "query_tokens": w.q_tokens, "generated": gen,
                               "ms_per_token": round(gen_ms, 4), "tokens_per_s": round(1e3 / gen_ms, 1),
                               "cache_gb_s": round(cache_bytes / (gen_ms * 1e-3) / 1e9, 1),
                               "graph_ms_per_token": round(gen_graph_ms, 4),
                               "graph_cache_gb_s": round(cache_bytes / (gen_graph_ms * 1e-3) / 1e9, 1)}
        del gq, gk, gv, ks, vs, toks

        # summary scorers on the 128K and 1M token ids (selection alone)
        sc = {}
        for wl in (WORKLOAD, workloads.SCALE_1M):
            idd = torch.from_numpy(wl.token_ids()).to(dev)
            sws = torch.empty(P.pa_select_workspace_size(wl.L, wl.vocab, wl.block, wl.chunk), dtype=torch.uint8,
                              device=dev)
            for name, method in (("max_idf", P.PA_SCORE_MAX_IDF), ("mean_idf", P.PA_SCORE_MEAN_IDF),
                                 ("entropy", P.PA_SCORE_ENTROPY), ("bm25", P.PA_SCORE_BM25),
                                 ("evenly_spaced", P.PA_SCORE_EVENLY_SPACED)):
                def sel_call():
                    P.pulsar_select_summaries_scored(idd, wl.vocab, wl.block, wl.chunk, wl.k_chunks, method,
                                                     ws=sws)
                for _ in range(3):
                    sel_call()
                torch.cuda.synchronize()
                a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a0.record()
                for _ in range(10):
                    sel_call()
                a1.record()
                torch.cuda.synchronize()
                sc[f"{wl.name}:{name}_us"] = round(a0.elapsed_time(a1) / 10 * 1e3, 1)
                require_ok(P, sws, f"selection {wl.name} {name}")
                # the same call captured once in a CUDA graph and replayed: the
                # GPU time without the Python / ctypes enqueue cost per call
                graph = torch.cuda.CUDAGraph()
                with torch.cuda.graph(graph):
                    sel_call()
                for _ in range(3):
                    graph.replay()
                torch.cuda.synchronize()
                a0.record()
                for _ in range(20):
                    graph.replay()
                a1.record()
                torch.cuda.synchronize()
                sc[f"{wl.name}:{name}_graph_us"] = round(a0.elapsed_time(a1) / 20 * 1e3, 1)
                del graph
        extra["selection_us"] = sc

    q2_bytes = 2.0 * w.L * w.hkv * w.d * 2
    # the query's roofline: the slower of streaming K/V at the measured copy
    # bandwidth and its QK^T + PV work at the measured burst bf16 peak
    q2_roof_ms = max(q2_bytes / (peaks["hbm_gbs"] * 1e9),
                     4.0 * w.d * w.hq * w.q_tokens * w.L / (peaks["bf16_tflops"] * 1e12)) * 1e3
    clocks = clk.summary()
    line = {
        "metric": METRIC, "value": round(tokens_per_s, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": round(ms, 3), "higher_is_better": True,
        "scaling": "strong" if hosts_layout else "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": w.name, "L": w.L, "block": w.block, "n_blocks": w.n_blocks, "hq": w.hq,
                   "hkv": w.hkv, "d": w.d, "sink": w.sink, "chunk": w.chunk,
                   "summary_tokens": w.k_chunks * w.chunk, "q_tokens": w.q_tokens,
                   "rope_theta": w.rope_theta,
                   "layout": args.layout,
                   "per_rank": (f"hosts [{h0}, {h1}) of one shared 128K sequence, then the Phase-2 NCCL all-gather"
                                if hosts_layout else "one independent 128K sequence"),
                   "l2": "inputs larger than L2 (Q alone is 1 GiB)"},
        "clocks": clocks,
        "e2e": {"value": round(e2e_rate, 1), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 3)},
        "gpu_launches": step.launches() * K,
        "roofline": {"bound": "tensor", "kernel": "phase-1 attention", "achieved": round(attn_tf, 1),
                     "peak": peak_tf, "unit": "TFLOP/s", "frac": round(attn_tf / peak_tf, 4),
                     "peak_kind": f"{peak_kind} bf16 burst",
                     "traffic": recorded_traffic("phase1_tc_kernel", w.name),
                     "kernel_ms": round(attn_ms, 3), "flop_per_launch": flops,
                     "frac_of_nominal_dense_bf16": round(attn_tf / NOMINAL_BF16_TFLOPS, 4),
                     "frac_of_sustained": round(attn_tf / peaks["bf16_tflops_sustained"], 4)},
        "phase1_encode": {"selection_ms": round(sel_ms, 4), "encode_ms": round(enc_ms, 3),
                          "tokens_per_s": round(w.L / (enc_ms * 1e-3), 1),
                          "with_selection_tokens_per_s": round(w.L / ((sel_ms + enc_ms) * 1e-3), 1),
                          "note": "encode = position map + RoPE + attention over all hosts"},
        "phase1": {"attn_ms": round(attn_ms, 3), "tflop": round(flops / 1e12, 3),
                   "tflop_s": round(attn_tf, 1)},
        "phase2_query": {"kernel": "phase2_tc_kernel", "kernel_ms": round(p2_ms, 4), "kv_bytes": q2_bytes,
                         "traffic": recorded_traffic("phase2_tc_kernel", w.name + ":query64"),
                         "gb_s": round(q2_bytes / (p2_ms * 1e-3) / 1e9, 1),
                         "frac_hbm": round(q2_bytes / (p2_ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
                         "tflop_s": round(4.0 * w.d * w.hq * w.q_tokens * w.L / (p2_ms * 1e-3) / 1e12, 1),
                         "roofline_ms": round(q2_roof_ms, 4), "frac_roofline": round(q2_roof_ms / p2_ms, 4),
                         "call_ms": round(p2_call_ms, 4)},
    }
    line.update(extra)
    return line


# --------------------------------------------------------------------------
# the oracle on the host cores (cpu_baseline leg and --impl reference)
# --------------------------------------------------------------------------
ORACLE_SAMPLE_ROWS = 512   # Phase-1 rows of the last host timed on the host cores (about 7 s on 16 cores)


def _oracle_threads():
    """Threads the oracle's numpy BLAS uses, and the host's logical cores."""
    from threadpoolctl import threadpool_info
    blas = max([i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"] + [1])
    return blas, os.cpu_count() or 1


class OracleSample:
    """The fp64 oracle timed on one fixed sample of a step, extrapolated.

    The sample is the same in every run (and in both the cpu_baseline leg
    and --impl reference): the whole Max-IDF selection; Phase 1 of the last
    (longest) host for ``n_rows`` rows evenly spaced over it, which the
    oracle evaluates against every column up to the last sampled row (after
    rotating those rows), extrapolated to the step's algorithmic Phase-1
    FLOPs by the FLOPs it executed; Phase 2 of one kv group of the 64-token
    query, times the number of kv groups.  The fp64 inputs are prepared once,
    untimed, and paged in by an untimed call on the last sampled row."""

    def __init__(self, w, n_rows=ORACLE_SAMPLE_ROWS):
        import oracle
        self.oracle, self.w = oracle, w
        self.ids = w.token_ids()
        q, k, v = w.qkv()
        self.qf = q.to(torch.float64).numpy()
        self.kf = k.to(torch.float64).numpy()
        self.vf = v.to(torch.float64).numpy()
        del q, k, v
        sel = oracle.select_summaries(self.ids, w.block, w.chunk, w.k_chunks, w.vocab)
        self.pos_last = oracle.host_positions(w.L, w.block, w.sink, w.chunk, sel)[-1]
        n = len(self.pos_last)
        self.rows = np.unique(np.linspace(0, n - 1, n_rows).round().astype(np.int64))
        self.kc, self.vc = oracle.retained_kv(self.kf[:, :1], self.vf[:, :1], w.rope_theta)   # one kv head
        self.qq = w.query().to(torch.float64).numpy()[:, :, :w.hq // w.hkv]
        oracle.phase1_encode(self.qf, self.kf, self.vf, [self.pos_last], w.rope_theta, [self.rows[-1:]])

    def run(self):
        """Returns (estimated step seconds, sample description)."""
        o, w = self.oracle, self.w
        t = time.perf_counter()
        sel = o.select_summaries(self.ids, w.block, w.chunk, w.k_chunks, w.vocab)
        t_sel = time.perf_counter() - t
        pos = o.host_positions(w.L, w.block, w.sink, w.chunk, sel)
        assert np.array_equal(pos[-1], self.pos_last)
        t = time.perf_counter()
        o.phase1_encode(self.qf, self.kf, self.vf, [pos[-1]], w.rope_theta, [self.rows])
        t_p1 = time.perf_counter() - t
        cols = int(self.rows.max()) + 1
        executed = 4.0 * w.d * w.hq * self.rows.size * cols    # QK^T and PV of every sampled row over `cols`
        total_flops = attn_flops(w)
        t_p1_est = t_p1 * total_flops / executed
        t = time.perf_counter()
        o.phase2_attend(self.qq, self.kc[None], self.vc[None], w.n_blocks, w.L, w.rope_theta)
        t_p2 = time.perf_counter() - t
        est = t_sel + t_p1_est + t_p2 * w.hkv
        desc = (f"full selection ({t_sel:.2f} s); Phase 1 of the last host for {self.rows.size} evenly spaced "
                f"rows against {cols} columns ({executed / 1e9:.0f} GFLOP executed of {total_flops / 1e12:.1f} "
                f"TFLOP, {t_p1:.1f} s, extrapolated by FLOPs); Phase 2 one kv group of {w.hkv} ({t_p2:.2f} s, "
                f"x{w.hkv})")
        return est, desc


def oracle_tiny_full():
    """The complete oracle run of the tiny workload (selection, Phase 1 of
    every row of every host, the 32-token query over its 4 shards): seconds,
    nothing extrapolated."""
    import oracle
    w = workloads.TINY
    t = time.perf_counter()
    ids = w.token_ids()
    sel = oracle.select_summaries(ids, w.block, w.chunk, w.k_chunks, w.vocab)
    pos = oracle.host_positions(w.L, w.block, w.sink, w.chunk, sel)
    q, k, v = (x.to(torch.float64).numpy() for x in w.qkv())
    oracle.phase1_encode(q, k, v, pos, w.rope_theta)
    kc, vc = oracle.retained_kv(k, v, w.rope_theta)
    oracle.phase2_attend(w.query().to(torch.float64).numpy(), kc[None], vc[None], w.n_blocks, w.L, w.rope_theta)
    return time.perf_counter() - t


def cpu_baseline_record(est, desc, tiny_s):
    blas, nproc = _oracle_threads()
    w = WORKLOAD
    return {"value": round(w.L / est, 3), "unit": "tokens/s", "cores": blas, "nproc": nproc, "kind": "oracle",
            "sample": desc,
            "tiny_full": {"workload": workloads.TINY.name, "seconds": round(tiny_s, 3),
                          "tokens_per_s": round(workloads.TINY.L / tiny_s, 1), "extrapolated": False}}


def run_reference(args):
    w = WORKLOAD
    sample = OracleSample(w)
    ests, desc = [], ""
    for _ in range(args.warmup):
        sample.run()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        est, desc = sample.run()
        ests.append(est)
    sample_ms = (time.perf_counter() - t0) / max(args.steps, 1) * 1e3
    est = statistics.mean(ests)
    value = w.L / est
    rec = cpu_baseline_record(est, desc + f"; mean of {args.steps} runs of the same sample", oracle_tiny_full())
    return {"impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "tokens/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(sample_ms, 1),
            "extrapolated_ms_per_full_step": round(est * 1e3, 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": w.name, "L": w.L, "block": w.block,
                       "note": "each timed step runs the fixed oracle sample (ms_per_step is its wall time); "
                               "value extrapolates it to the whole 128K step "
                               "(extrapolated_ms_per_full_step)"},
            "cpu_baseline": rec,
            "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def run_profile_case(name, steps, warmup):
    """One kernel family on a small workload, for ncu captures:
    phase1-32k (Pulsar Phase 1 incl. its RoPE prepass, 32K shape),
    decode-128k / decode-16k (Phase-2 decode, 16 queries over a 128K / 16K
    cache in 8 shards), query-128k (Phase-2 64-token query), select-1m
    (Max-IDF selection over the 1M-token ids).  Prints one JSON line with the
    mean call time."""
    from long_context_blockwise_max_b200 import pulsar as P
    dev = torch.device("cuda", 0)
    if name == "phase1-32k":
        w = workloads.LLAMA_32K
        q, k, v = w.qkv(device=dev)
        sel, _, _, _ = P.pulsar_select_summaries(torch.from_numpy(w.token_ids()).to(dev), w.vocab, w.block,
                                                 w.chunk, w.k_chunks)
        out = P.pulsar_phase1_encode(q, k, v, w.rope_theta, w.block, w.sink, w.chunk, w.k_chunks, sel)
        o, lse, kr, vr, _, ws = out

        def call():
            P.pulsar_phase1_encode(q, k, v, w.rope_theta, w.block, w.sink, w.chunk, w.k_chunks, sel, o=o, lse=lse,
                                   k_ret=kr, v_ret=vr, ws=ws)
    elif name in ("decode-128k", "decode-16k"):
        w = DECODE
        T = w.decode_T if name == "decode-128k" else 16384
        q = workloads.normal((w.decode_batch, 1, w.hq, w.d), workloads.SEED_QUERY, w.dtype, dev)
        kc = workloads.normal((w.decode_batch, T, w.hkv, w.d), workloads.SEED_KC, w.dtype, dev)
        vc = workloads.normal((w.decode_batch, T, w.hkv, w.d), workloads.SEED_VC, w.dtype, dev)
        o, lse, _, _, ws = P.star_phase2_attend(q, kc, vc, w.decode_shards, T, w.rope_theta)

        def call():
            P.star_phase2_attend(q, kc, vc, w.decode_shards, T, w.rope_theta, o=o, lse=lse, ws=ws)
    elif name == "query-128k":
        w = WORKLOAD
        q = w.query(device=dev)
        kc = workloads.normal((1, w.L, w.hkv, w.d), workloads.SEED_KC, w.dtype, dev)
        vc = workloads.normal((1, w.L, w.hkv, w.d), workloads.SEED_VC, w.dtype, dev)
        o, lse, _, _, ws = P.star_phase2_attend(q, kc, vc, w.n_blocks, w.L, w.rope_theta)

        def call():
            P.star_phase2_attend(q, kc, vc, w.n_blocks, w.L, w.rope_theta, o=o, lse=lse, ws=ws)
    elif name == "select-1m":
        w = workloads.SCALE_1M
        idd = torch.from_numpy(w.token_ids()).to(dev)
        sel, _, _, _ = P.pulsar_select_summaries(idd, w.vocab, w.block, w.chunk, w.k_chunks)
        sws = torch.empty(P.pa_select_workspace_size(w.L, w.vocab, w.block, w.chunk), dtype=torch.uint8,
                          device=dev)

        def call():
            P.pulsar_select_summaries(idd, w.vocab, w.block, w.chunk, w.k_chunks, sel=sel, ws=sws)
    else:
        raise SystemExit(f"unknown profile case {name}")
    for _ in range(warmup):
        call()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        call()
    e1.record()
    torch.cuda.synchronize()
    print(json.dumps({"profile_case": name, "steps": steps, "ms_per_call": e0.elapsed_time(e1) / max(steps, 1)}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--headline-only", action="store_true", help="skip the side measurements")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--layout", default=None, choices=["sequences", "hosts"],
                    help="hosts (the default with several GPUs): the hosts of one sequence spread over the ranks, "
                         "then the Phase-2 all-gather over NCCL (strong scaling); sequences (the default on one "
                         "GPU, where both are the same work): one independent sequence per rank (weak scaling)")
    ap.add_argument("--profile-case", default=None,
                    help="run one kernel family on a small workload (phase1-32k, decode-16k, decode-128k, query-128k, select-1m)")
    args = ap.parse_args()
    if args.profile_case:
        run_profile_case(args.profile_case, args.steps, args.warmup)
        return

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.layout is None:
        args.layout = "hosts" if world > 1 else "sequences"
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return
    dist_on = world > 1
    group_on = dist_on or args.layout == "hosts"
    if group_on:
        import datetime
        torch.cuda.set_device(local_rank)
        if not dist_on:   # the hosts layout on one GPU: a process group of one rank
            import socket
            with socket.socket() as sk:
                sk.bind(("127.0.0.1", 0))
                os.environ.setdefault("MASTER_PORT", str(sk.getsockname()[1]))
            os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
            os.environ.setdefault("RANK", "0")
            os.environ.setdefault("WORLD_SIZE", "1")
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local_rank))
    try:
        line = run_ours(args, rank, world, local_rank, dist_on)
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            est, desc = OracleSample(WORKLOAD).run()
            line["cpu_baseline"] = cpu_baseline_record(est, desc, oracle_tiny_full())
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if group_on:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
