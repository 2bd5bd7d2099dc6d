"""Benchmark of the KDA hot path on B200: one JSON line per run.

A step is one pass of the whole hot path over one batch of synthetic input:
  1. kda_prefill  - chunked prefill of 8192 tokens x 64 heads, d_k = d_v = 128,
                    chunk 64, bf16 q/k/v/o, fp32 state, snapshots every 256 tokens;
  2. kda_decode   - one token for 512 sequences x 64 heads against fp32 states;
  3. kda_verify   - 1..8 draft tokens per sequence (seeded uniform), writing the
                    state after every token;
  4. kda_snapshot - commit the state of each sequence's last accepted token
                    (seeded acceptance) into its live slot;
  5. kda_verify_commit - the same speculative step with the commit fused in: the
                    verify batch above, accepted as in 4, is replayed into the live
                    state, then the next 1..8 draft tokens run with outputs only.
The tiny fp32 workload, the 32-sequence ragged batch and the 1M-token segmented
prefill are timed in the same run, each on its own, under "components".
Inputs are seeded (synth.py) and resident in HBM before timing; every input set
is larger than the 126 MB L2 (prefill 0.94 GB, decode 2.1 GB, verify 12 GB), so
no L2 flush is needed between steps.

`value` is prefill tokens per second (tokens of all 64 heads), summed over
ranks; the decode and verify rows are reported in state-steps per second (one
(sequence, head) state advanced by one token) under "components". Times are
CUDA events on the launching stream; for N > 1 the max over ranks. With
--gpus N > 1 the ranks are independent replicas (the layer has no exchange).

--impl reference times the fp64 CPU oracle (the test oracle, untuned) on a
bounded sample of the same prefill workload, on the host cores.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time
from pathlib import Path

import numpy as np
import torch

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

import synth  # noqa: E402

METRIC = "KDA prefill tok/s + decode state-steps/s on 1 B200; % of TC/HBM roofline"
H, D, C = 64, 128, 64
PREFILL_T = 8192
SNAP = 256
E2E_WIN = 1024          # tokens per window of the end-to-end prefill (a multiple of SNAP)
N_SEQ = 512
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}


# ----------------------------------------------------------------------------
def load_peaks():
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        d = json.loads(p.read_text())
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return {**FALLBACK, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def _src_hash(files):
    h = hashlib.sha256()
    for f in files:
        h.update((ROOT / "hybrid_linear_attention_04_b200" / "csrc" / f).read_bytes())
    return h.hexdigest()[:16]


def ncu_traffic(kernel, read_units, write_units):
    """DRAM bytes per launch (read + write) of `kernel` scaled from the committed
    ncu capture by the units this launch processes, or None when the capture is
    missing or was taken on other kernel sources."""
    p = ROOT / "profiles" / "dram_traffic.json"
    if not p.exists():
        return None
    d = json.loads(p.read_text())
    k = d.get("kernels", {}).get(kernel)
    if not k or _src_hash(d["sources"][kernel]) != k["src_hash"]:
        return None
    return int(k["read"] / k["read_units"] * read_units + k["write"] / k["write_units"] * write_units)


class ClockSampler:
    """Samples SM clock, max clock, power and clock-event reasons through NVML
    every ~5 ms in a background thread while the timed region runs (read-only;
    no setting of the GPU is changed)."""

    def __init__(self, dev):
        self.dev = dev
        self.samples = []
        self.thread = None
        self.stop = False

    def _handle(self):
        import pynvml
        pynvml.nvmlInit()
        try:
            pr = torch.cuda.get_device_properties(self.dev)
            bus = f"{pr.pci_domain_id:08x}:{pr.pci_bus_id:02x}:{pr.pci_device_id:02x}.0"
            return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
            idx = int(vis.split(",")[self.dev.index or 0]) if vis and vis.split(",")[0].isdigit() else (self.dev.index or 0)
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(idx)

    def _run(self):
        nv, h = self.nv, self.h
        names = {"hw_slowdown": nv.nvmlClocksEventReasonHwSlowdown,
                 "hw_thermal_slowdown": nv.nvmlClocksEventReasonHwThermalSlowdown,
                 "sw_thermal_slowdown": nv.nvmlClocksEventReasonSwThermalSlowdown,
                 "sw_power_cap": nv.nvmlClocksEventReasonSwPowerCap,
                 "hw_power_brake": nv.nvmlClocksEventReasonHwPowerBrakeSlowdown}
        self.sm_max = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        while not self.stop:
            try:
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                self.samples.append((sm, pw, [n for n, b in names.items() if rs & b]))
            except Exception:
                pass
            time.sleep(0.005)

    def __enter__(self):
        import threading
        try:
            self.nv, self.h = self._handle()
        except Exception:
            return self
        self.thread = threading.Thread(target=self._run, daemon=True)
        self.thread.start()
        while not self.samples and self.thread.is_alive():
            time.sleep(0.001)
        return self

    def __exit__(self, *a):
        self.stop = True
        if self.thread is not None:
            self.thread.join(timeout=5)

    def summary(self):
        if not self.samples:
            return None
        sm = [x[0] for x in self.samples]
        reasons = sorted({r for x in self.samples for r in x[2]})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": getattr(self, "sm_max", None),
                "reasons": reasons, "samples": len(sm),
                "power_w_max": round(max(x[1] for x in self.samples), 1)}


# ----------------------------------------------------------------------------
def prefill_bytes(T, n_seq, n_snap, with_state_in):
    per_tok = H * (3 * D * 2 + D * 2 + D * 4 + 4)     # q,k,v,o bf16 + g fp32 + beta
    state = H * D * D * 4
    return T * per_tok + (n_snap + n_seq * (2 if with_state_in else 1)) * state


def prefill_flops(T):
    # chunk form per token-head, d_k = d_v = d, chunk C (causal halves):
    # 6 d^2 (S_0 products and state update) + C (3 d_k + 2 d_v) + C^2 / 3
    return T * H * (6 * D * D + C * (3 * D + 2 * D) + C * C / 3)


def decode_bytes(n):
    return n * H * (2 * D * D * 4 + 3 * D * 2 + D * 4 + 4 + D * 2)


def verify_bytes(n_seq, n_tok):
    return n_seq * H * D * D * 4 + n_tok * H * (D * D * 4 + 3 * D * 2 + D * 4 + 4 + D * 2)


def commit_bytes(n):
    return n * H * D * D * 4 * 2


def verify_commit_bytes(n_seq, n_written, n_replayed, n_tok):
    """State read once per sequence and written once where a commit happened; replayed
    tokens' k, v (bf16), g, beta; drafted tokens' q, k, v, o (bf16), g, beta."""
    return (n_seq + n_written) * H * D * D * 4 + n_replayed * H * (2 * D * 2 + D * 4 + 4) \
        + n_tok * H * (4 * D * 2 + D * 4 + 4)


class Workload:
    """The serving-step workload, resident on one device."""

    def __init__(self, dev, prefill_path="split", T=PREFILL_T, n_seq=N_SEQ):
        from hybrid_linear_attention_04_b200 import kda as K
        self.K = K
        self.dev = dev
        self.T, self.n_seq = T, n_seq
        x = synth.token_inputs(1001, T, H, D, D, io="bf16")
        self.host_prefill = x
        self.p = {k: v.to(dev) for k, v in x.items()}
        self.cu = np.array([0, T], dtype=np.int32)
        offs, _ = K.kda_snapshot_plan(self.cu, None, SNAP)
        self.n_snap = int(offs[-1])
        self.p_o = torch.empty((T, H, D), dtype=torch.bfloat16, device=dev)
        self.p_sout = torch.empty((1, H, D, D), device=dev)
        self.p_snaps = torch.empty((self.n_snap, H, D, D), device=dev)
        # "split": two launches through a workspace; "fused": one launch, no workspace
        self.p_ws = None
        if prefill_path == "split":
            nbytes = K.kda_prefill_workspace_size(self.p["q"], self.p["v"], self.cu, C)
            self.p_ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
        # decode + verify
        self.pool = synth.states(1002, n_seq, H, D, D, std=0.1).to(dev)
        self.slots = torch.arange(n_seq, dtype=torch.int32, device=dev)
        y = synth.token_inputs(1002, n_seq, H, D, D, io="bf16")
        self.d = {k: v.to(dev) for k, v in y.items()}
        self.d_o = torch.empty((n_seq, H, D), dtype=torch.bfloat16, device=dev)
        lens = synth.draft_lengths(1002, n_seq, 1, 8)
        self.cu_draft = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
        self.n_tok = int(self.cu_draft[-1])
        z = synth.token_inputs(1002, self.n_tok, H, D, D, io="bf16", t0=n_seq)
        self.v = {k: v.to(dev) for k, v in z.items()}
        self.v_o = torch.empty((self.n_tok, H, D), dtype=torch.bfloat16, device=dev)
        self.ts = torch.empty((self.n_tok, H, D, D), device=dev)
        acc = synth.randint(1002, "misc", n_seq, 0, 8)
        src, dst = [], []
        for s in range(n_seq):
            a = min(acc[s], lens[s])
            if a > 0:
                src.append(int(self.cu_draft[s]) + a - 1)
                dst.append(s)
        self.c_src = torch.tensor(src, dtype=torch.int64, device=dev)
        self.c_dst = torch.tensor(dst, dtype=torch.int64, device=dev)
        self.n_commit = len(src)
        # verify with the previous step's commit fused in: the previous batch is the
        # verify batch above with the same seeded acceptance; this step's drafts are the
        # next 1..8 tokens per sequence of the same streams
        self.vc_acc = [min(acc[s], lens[s]) for s in range(n_seq)]
        self.vc_acc_d = torch.tensor(self.vc_acc, dtype=torch.int32, device=dev)
        lens2 = synth.draft_lengths(1002, n_seq, 1, 8, start=n_seq)
        self.vc_cu = np.concatenate([[0], np.cumsum(lens2)]).astype(np.int32)
        self.vc_tok = int(self.vc_cu[-1])
        z2 = synth.token_inputs(1002, self.vc_tok, H, D, D, io="bf16", t0=n_seq + self.n_tok)
        self.vc = {k: v.to(dev) for k, v in z2.items()}
        self.vc_o = torch.empty((self.vc_tok, H, D), dtype=torch.bfloat16, device=dev)

    def prefill(self):
        K, p = self.K, self.p
        K.kda_prefill(p["q"], p["k"], p["v"], p["g"], p["beta"], self.cu, self.p_o,
                      state_out=self.p_sout, snap_interval=SNAP, snapshots=self.p_snaps, chunk=C,
                      workspace=self.p_ws)

    def decode(self):
        d = self.d
        self.K.kda_decode(d["q"], d["k"], d["v"], d["g"], d["beta"], self.slots, self.pool, self.d_o)

    def verify(self):
        v = self.v
        self.K.kda_verify(v["q"], v["k"], v["v"], v["g"], v["beta"], self.cu_draft, self.slots,
                          self.pool, self.ts, self.v_o)

    def commit(self):
        self.K.kda_snapshot(self.c_src, self.c_dst, self.ts, self.pool)

    def verify_commit(self):
        c = self.vc
        self.K.kda_verify_commit(self.v, self.vc_acc_d, self.cu_draft, c["q"], c["k"], c["v"],
                                 c["g"], c["beta"], self.vc_cu, self.slots, self.pool, self.vc_o)


def dist_setup(n_gpus):
    if n_gpus > 1 or int(os.environ.get("WORLD_SIZE", "1")) > 1:
        import datetime
        import torch.distributed as dist
        local = int(os.environ.get("LOCAL_RANK", "0"))
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        return dist, dist.get_rank(), dist.get_world_size(), local
    return None, 0, 1, 0


def max_over_ranks(dist, x, dev):
    if dist is None:
        return x
    t = torch.tensor(x, dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def cpu_baseline_prefill(tokens, heads):
    """The oracle, as it stands, on `tokens` x `heads` of the prefill workload."""
    from oracle import native
    x = synth.token_inputs(1001, tokens, H, D, D, io="bf16")
    sl = {k: v[:, :heads].contiguous() for k, v in x.items()}
    native.load()
    t0 = time.perf_counter()
    native.oracle_sequence(sl["q"], sl["k"], sl["v"], sl["g"], sl["beta"], None, None, 0, SNAP,
                           out_dtype=np.float32)
    dt = time.perf_counter() - t0
    return dt, native.max_threads()


# ----------------------------------------------------------------------------
def run_ours(args):
    dist, rank, world, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    from hybrid_linear_attention_04_b200 import build as kbuild
    if rank == 0:
        kbuild.build()
    if dist is not None:
        dist.barrier()
    from hybrid_linear_attention_04_b200 import kda as K
    wl = Workload(dev, args.prefill_path, args.prefill_tokens, args.decode_seqs)
    stream = torch.cuda.current_stream(dev)
    comps = ["prefill", "decode", "verify", "commit", "verify_commit"]
    fns = [wl.prefill, wl.decode, wl.verify, wl.commit, wl.verify_commit]

    def step(ev=None):
        for i, f in enumerate(fns):
            if ev is not None:
                ev[i][0].record(stream)
            f()
            if ev is not None:
                ev[i][1].record(stream)

    for _ in range(args.warmup):
        step()
    st = K.kda_check_device_status()
    if st != 0:
        raise RuntimeError(f"device status {K.kda_status_string(st)} after warm-up")
    evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in comps]
           for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize(dev)
    launches0 = K.kda_launch_count()
    with ClockSampler(dev) as clk:
        t_start.record(stream)
        for s in range(args.steps):
            step(evs[s])
        t_end.record(stream)
        torch.cuda.synchronize(dev)
    launches = K.kda_launch_count() - launches0
    if dist is not None:
        dist.barrier()
    st = K.kda_check_device_status()
    if st != 0:
        raise RuntimeError(f"device status {K.kda_status_string(st)} after timing")
    total_ms = t_start.elapsed_time(t_end)
    comp_ms = [sum(evs[s][i][0].elapsed_time(evs[s][i][1]) for s in range(args.steps)) / args.steps
               for i in range(len(comps))]
    vals = max_over_ranks(dist, [total_ms] + comp_ms, dev)
    total_ms, comp_ms = vals[0], vals[1:]

    # end to end through the same C-ABI call, host buffers: every step copies its prefill
    # inputs from pinned memory, runs the prefill and reads its outputs back. The step runs
    # in windows of E2E_WIN tokens on three streams (H2D, compute, D2H), so that the copies
    # in both directions overlap the kernels and each other; each window hands its state to
    # the next in fp32 (the chunks are those of one call, so are the results).
    hp = {k: v.pin_memory() for k, v in wl.host_prefill.items()}
    ho = torch.empty(wl.p_o.shape, dtype=wl.p_o.dtype).pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in hp.values())
    d2h = ho.numel() * ho.element_size()
    s_h2d, s_d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    wins = [(a, min(wl.T, a + E2E_WIN)) for a in range(0, wl.T, E2E_WIN)]
    win_states = [torch.empty_like(wl.p_sout) for _ in range(2)]
    win_ws = None
    if wl.p_ws is not None:
        win_cu = np.array([0, E2E_WIN], dtype=np.int32)
        win_ws = torch.empty(K.kda_prefill_workspace_size(wl.p["q"][:E2E_WIN], wl.p["v"][:E2E_WIN],
                                                          win_cu, C), dtype=torch.uint8, device=dev)
    prev = {"done": [None] * len(wins), "read": [None] * len(wins)}

    def e2e_step():
        p = wl.p
        done, read = [], []
        for w, (a, b) in enumerate(wins):
            with torch.cuda.stream(s_h2d):
                if prev["done"][w] is not None:          # last step's kernels have read window w
                    s_h2d.wait_event(prev["done"][w])
                for k in hp:
                    p[k][a:b].copy_(hp[k][a:b], non_blocking=True)
                landed = torch.cuda.Event()
                landed.record(s_h2d)
            stream.wait_event(landed)
            if prev["read"][w] is not None:              # last step's outputs of window w are out
                stream.wait_event(prev["read"][w])
            last = w == len(wins) - 1
            K.kda_prefill(p["q"][a:b], p["k"][a:b], p["v"][a:b], p["g"][a:b], p["beta"][a:b],
                          np.array([0, b - a], dtype=np.int32), wl.p_o[a:b],
                          state_out=wl.p_sout if last else win_states[w % 2],
                          state_in=None if w == 0 else win_states[(w - 1) % 2],
                          start_pos=np.array([a], dtype=np.int64), snap_interval=SNAP,
                          snapshots=wl.p_snaps[a // SNAP:b // SNAP], chunk=C, workspace=win_ws)
            ev = torch.cuda.Event()
            ev.record(stream)
            done.append(ev)
            s_d2h.wait_event(ev)
            with torch.cuda.stream(s_d2h):
                ho[a:b].copy_(wl.p_o[a:b], non_blocking=True)
                out = torch.cuda.Event()
                out.record(s_d2h)
            read.append(out)
        prev["done"], prev["read"] = done, read
        stream.wait_stream(s_d2h)                        # the step ends with its outputs on the host

    e2e_step()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    s_h2d.wait_event(e0)
    for _ in range(args.steps):
        e2e_step()
    stream.wait_stream(s_h2d)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(dist, [e0.elapsed_time(e1) / args.steps], dev)[0]
    # the windows' outputs against one call on the same inputs (outside the timed region)
    wl.prefill()
    torch.cuda.synchronize(dev)
    e2e_same = bool(torch.equal(wl.p_o.cpu(), ho))

    # the other workloads, each timed on its own (CUDA events over `steps` calls)
    peaks = load_peaks()
    extra = {}
    if not args.serving_only:
        del wl.p_ws, wl.ts
        torch.cuda.empty_cache()
        extra["tiny"] = bench_tiny(K, dev, args.steps, args.warmup)
        extra.update(bench_frontend(K, dev, args.steps, args.warmup, peaks))
        extra["ragged"] = bench_ragged(K, dev, args.steps, args.warmup, peaks)
        torch.cuda.empty_cache()
        extra["long"] = bench_long(K, dev, max(3, args.steps // 4), args.warmup, peaks)
        torch.cuda.empty_cache()
        for name in extra:
            key = "ms"
            extra[name][key] = max_over_ranks(dist, [extra[name][key]], dev)[0]

    result = None
    if rank == 0:
        hbm = peaks["hbm_gbs"]
        comp = {}
        units = {
            "prefill": (wl.T, "tok/s", prefill_bytes(wl.T, 1, wl.n_snap, False)),
            "decode": (wl.n_seq * H, "state-steps/s", decode_bytes(wl.n_seq)),
            "verify": (wl.n_tok * H, "state-steps/s", verify_bytes(wl.n_seq, wl.n_tok)),
            "commit": (wl.n_commit, "states/s", commit_bytes(wl.n_commit)),
            "verify_commit": ((sum(wl.vc_acc) + wl.vc_tok) * H, "state-steps/s",
                              verify_commit_bytes(wl.n_seq, sum(1 for a in wl.vc_acc if a > 0),
                                                  sum(wl.vc_acc), wl.vc_tok)),
        }
        for name, ms in zip(comps, comp_ms):
            n_units, unit, byts = units[name]
            gbs = byts / (ms * 1e-3) / 1e9
            comp[name] = {"ms": round(ms, 4), "value": world * n_units / (ms * 1e-3), "unit": unit,
                          "algorithmic_bytes": byts, "achieved_gbs": round(gbs, 1),
                          "hbm_frac": round(gbs / hbm, 4)}
        pf = prefill_flops(wl.T)
        comp["prefill"]["algorithmic_flops"] = pf
        comp["prefill"]["tc_frac"] = round(pf / (comp_ms[0] * 1e-3) / (peaks["bf16_tflops"] * 1e12), 4)
        comp["prefill"]["path"] = args.prefill_path
        for name, e in extra.items():
            if "tokens" in e:
                e["value"] = world * e["tokens"] / (e["ms"] * 1e-3)
            comp[name] = e
        dom = max(comps, key=lambda c: comp[c]["ms"])
        pk = ["prefill_prep_kernel", "prefill_chain_kernel"] if args.prefill_path == "split" \
            else ["prefill_tc_kernel"]
        knames = {"prefill": pk, "decode": ["decode_kernel"], "verify": ["spec_kernel<verify>"],
                  "commit": ["snapshot_kernel"], "verify_commit": ["spec_kernel<verify+commit>"]}[dom]
        kname = "+".join(knames)
        tr_units = {"prefill": (wl.T * H, wl.T * H), "decode": (wl.n_seq * H, wl.n_seq * H),
                    "verify": (wl.n_seq * H, wl.n_tok * H), "commit": (wl.n_commit, wl.n_commit),
                    "verify_commit": (wl.n_seq * H, wl.n_seq * H)}[dom]
        trs = [ncu_traffic(k, *tr_units) for k in knames]
        tr = None if any(t is None for t in trs) else sum(trs)
        roof = {"bound": "hbm", "kernel": kname, "achieved": comp[dom]["achieved_gbs"],
                "peak": hbm, "unit": "GB/s", "frac": comp[dom]["hbm_frac"],
                "traffic": tr, "peak_source": peaks["source"]}
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            tok = args.cpu_tokens
            dt, cores = cpu_baseline_prefill(tok, H)
            cpu = {"value": tok / dt, "unit": "tok/s", "cores": cores, "kind": "oracle",
                   "sample": f"fp64 token recurrence, first {tok} tokens x {H} heads of the "
                             f"prefill workload ({dt:.1f} s)"}
        clocks = clk.summary()
        result = {
            "metric": METRIC,
            "value": world * wl.T / (comp_ms[0] * 1e-3),
            "unit": "tok/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(total_ms / args.steps, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": {"workload": f"prefill {wl.T} tok x 64 heads (d=128, chunk 64, snapshots /256)"
                                   f" + decode/verify/commit {wl.n_seq} seq x 64 heads (drafts 1..8)",
                       "global_batch": world * (1 + wl.n_seq), "seq_len": wl.T,
                       "parallelism": f"replicas x{world}",
                       "l2": "inputs larger than L2 (no flush)"},
            "components": comp,
            "roofline": roof,
            "cpu_baseline": cpu,
            "e2e": {"value": world * wl.T / (e2e_ms * 1e-3), "unit": "tok/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "scope": f"prefill with pinned-host inputs and outputs, in windows of "
                             f"{E2E_WIN} tokens on H2D, compute and D2H streams",
                    "outputs_equal_one_call": e2e_same},
            "gpu_launches": launches,
            "clocks": clocks,
        }
        print(json.dumps(result), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return result


def prefill_bytes_general(T, n_seq, n_snap, n_state_in, io_bytes=2, d=D, heads=H):
    """Algorithmic bytes of one prefill call: q, k, v, o in the I/O type, g fp32, beta,
    snapshots, final states and the initial states read."""
    per_tok = heads * (4 * d * io_bytes + d * 4 + 4)
    return T * per_tok + (n_snap + n_seq + n_state_in) * heads * d * d * 4


def bench_tiny(K, dev, steps, warmup):
    """The tiny all-fp32 workload: B=1, H=2, T=64, d=32, chunk 16 (CUDA-core path)."""
    c = synth.WORKLOADS["tiny_fp32"]
    x = synth.token_inputs(c["seed"], c["T"], c["H"], c["d"], c["d"], io="fp32")
    xd = {k: v.to(dev) for k, v in x.items()}
    o = torch.empty_like(xd["v"])
    so = torch.empty((1, c["H"], c["d"], c["d"]), device=dev)
    cu = np.array([0, c["T"]], dtype=np.int32)
    n0 = K.kda_launch_count()
    K.kda_prefill(xd["q"], xd["k"], xd["v"], xd["g"], xd["beta"], cu, o, state_out=so,
                  chunk=c["chunk"], workspace=None)
    launches = K.kda_launch_count() - n0
    def call():
        K.kda_prefill(xd["q"], xd["k"], xd["v"], xd["g"], xd["beta"], cu, o, state_out=so,
                      chunk=c["chunk"], workspace=None)
    ms = time_calls(call, steps, warmup, dev)
    # the same call captured once in a CUDA graph and replayed: the device time per call
    # without the host's per-call work (argument checks, marshalling, launch)
    graph_us = None
    try:
        side = torch.cuda.Stream(device=dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(side):
            call()
        torch.cuda.current_stream(dev).wait_stream(side)
        torch.cuda.synchronize(dev)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for _ in range(10):
                call()
        graph_us = round(time_calls(graph.replay, max(3, steps // 10), warmup, dev) * 1e2, 2)
        del graph
    except Exception:                 # graph capture unavailable: report the eager time only
        graph_us = None
    byts = prefill_bytes_general(c["T"], 1, 0, 0, io_bytes=4, d=c["d"], heads=c["H"])
    return {"ms": round(ms, 5), "value": round(ms * 1e3, 2), "unit": "us/call",
            "graph_replay_us_per_call": graph_us,
            "tok_per_s": c["T"] / (ms * 1e-3), "algorithmic_bytes": byts,
            "bound": "latency (one CTA per head walks the chunks)", "launches_per_call": launches,
            "workload": "B=1, H=2, T=64, d=32, chunk 16, fp32 throughout, zero initial state"}


def bench_ragged(K, dev, steps, warmup, peaks):
    """The ragged packed prefill with prefix reuse: 32 sequences, lognormal lengths,
    half of them resuming from the GPU's own snapshot of a shared 16384-token prefix."""
    c = synth.WORKLOADS["ragged_prefix_32"]
    plan = synth.ragged_plan(c["seed"], c["n_seq"], c["mu"], c["sigma"], c["lo"], c["hi"],
                             c["prefix"], c["n_resume"], c["snap"])
    lens, start = plan["lens"], plan["start_pos"]
    n_seq, snap, P = len(lens), c["snap"], c["prefix"]
    # the shared prefix, prefilled once (untimed), gives the resumers' initial states
    xp = synth.token_inputs_device(c["seed"] + 1, P, H, D, D, io="bf16", device=dev)
    cup = np.array([0, P], dtype=np.int32)
    po = torch.empty((P, H, D), dtype=torch.bfloat16, device=dev)
    psn = torch.empty((P // snap, H, D, D), device=dev)
    K.kda_prefill(xp["q"], xp["k"], xp["v"], xp["g"], xp["beta"], cup, po, snap_interval=snap,
                  snapshots=psn, chunk=C)
    s0 = torch.zeros((n_seq, H, D, D), device=dev)
    res = plan["resumers"]
    K.kda_snapshot(torch.tensor([plan["resume_block"][s] - 1 for s in res], dtype=torch.int64,
                                device=dev),
                   torch.tensor(res, dtype=torch.int64, device=dev), psn, s0)
    del xp, po, psn
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = int(cu[-1])
    xd = synth.token_inputs_device(c["seed"], T, H, D, D, io="bf16", device=dev)
    o = torch.empty((T, H, D), dtype=torch.bfloat16, device=dev)
    so = torch.empty_like(s0)
    offs, _ = K.kda_snapshot_plan(cu, start, snap)
    sn = torch.empty((int(offs[-1]), H, D, D), device=dev)
    ws = torch.empty(K.kda_prefill_workspace_size(xd["q"], xd["v"], cu, C), dtype=torch.uint8,
                     device=dev)

    def call():
        K.kda_prefill(xd["q"], xd["k"], xd["v"], xd["g"], xd["beta"], cu, o, state_out=so,
                      state_in=s0, start_pos=start, snap_interval=snap, snapshots=sn, chunk=C,
                      workspace=ws)
    n0 = K.kda_launch_count()
    call()
    launches = K.kda_launch_count() - n0
    ms = time_calls(call, steps, warmup, dev)
    byts = prefill_bytes_general(T, n_seq, int(offs[-1]), n_seq)
    flops = prefill_flops(T)
    st = K.kda_check_device_status()
    if st != 0:
        raise RuntimeError(f"ragged workload: device status {K.kda_status_string(st)}")
    return {"ms": round(ms, 4), "value": T / (ms * 1e-3), "unit": "tok/s", "tokens": T,
            "algorithmic_bytes": byts, "achieved_gbs": round(byts / (ms * 1e-3) / 1e9, 1),
            "hbm_frac": round(byts / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
            "algorithmic_flops": flops,
            "tc_frac": round(flops / (ms * 1e-3) / (peaks["bf16_tflops"] * 1e12), 4),
            "launches_per_call": launches, "path": "split",
            "workload": f"{n_seq} sequences ({T} tokens) x 64 heads, lognormal(ln 4096, 1) "
                        f"lengths clipped to [512, 65536], {len(res)} resuming from snapshots "
                        f"of a shared {P}-token prefix, snapshots /{snap}"}


def bench_long(K, dev, steps, warmup, peaks):
    """The long-context prefill: 1,048,576 tokens as 16 calls of 65,536 with the state
    handed across calls and snapshots every 4096 tokens; one pass = 16 calls."""
    c = synth.WORKLOADS["long_1m"]
    seg, n_seg, snap = c["segment"], c["T"] // c["segment"], c["snap"]
    segs = [synth.token_inputs_device(c["seed"], seg, H, D, D, io="bf16", t0=i * seg, device=dev)
            for i in range(n_seg)]
    o = torch.empty((seg, H, D), dtype=torch.bfloat16, device=dev)
    st = [torch.empty((1, H, D, D), device=dev) for _ in range(2)]
    sn = torch.empty((c["T"] // snap, H, D, D), device=dev)
    cu = np.array([0, seg], dtype=np.int32)
    ws = torch.empty(K.kda_prefill_workspace_size(segs[0]["q"], segs[0]["v"], cu, C),
                     dtype=torch.uint8, device=dev)
    per = seg // snap

    def one_pass():
        for i in range(n_seg):
            xd = segs[i]
            K.kda_prefill(xd["q"], xd["k"], xd["v"], xd["g"], xd["beta"], cu, o,
                          state_out=st[(i + 1) % 2], state_in=st[i % 2] if i else None,
                          start_pos=[i * seg], snap_interval=snap, snapshots=sn[i * per:(i + 1) * per],
                          chunk=C, workspace=ws)
    n0 = K.kda_launch_count()
    one_pass()
    launches = K.kda_launch_count() - n0
    ms = time_calls(one_pass, steps, warmup, dev)
    T = c["T"]
    byts = prefill_bytes_general(T, n_seg, T // snap, n_seg - 1)
    flops = prefill_flops(T)
    stt = K.kda_check_device_status()
    if stt != 0:
        raise RuntimeError(f"long workload: device status {K.kda_status_string(stt)}")
    return {"ms": round(ms, 3), "value": T / (ms * 1e-3), "unit": "tok/s", "tokens": T,
            "algorithmic_bytes": byts, "achieved_gbs": round(byts / (ms * 1e-3) / 1e9, 1),
            "hbm_frac": round(byts / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
            "algorithmic_flops": flops,
            "tc_frac": round(flops / (ms * 1e-3) / (peaks["bf16_tflops"] * 1e12), 4),
            "launches_per_pass": launches, "path": "split",
            "workload": "1,048,576 tokens x 64 heads as 16 calls of 65,536 (state handed "
                        "across calls), snapshots /4096; one pass = 16 calls"}


def bench_frontend(K, dev, steps, warmup, peaks):
    """The q/k front-end (short conv, Swish, L2): kda_qk_frontend over the 8192-token
    prefill workload (raw q, k; conv states carried and snapshotted every 256 tokens),
    and kda_decode_conv, the decode step with the front-end fused in, on 512 x 64 states."""
    taps = 4
    T, n_seq = PREFILL_T, N_SEQ
    raw = synth.raw_qk(1001, T, H, D, io="bf16")
    rd = {k: v.to(dev) for k, v in raw.items()}
    wq, wk = (w.to(dev) for w in synth.conv_weights(1001, H, D, taps))
    qo, ko = torch.empty_like(rd["q"]), torch.empty_like(rd["k"])
    cu = np.array([0, T], dtype=np.int32)
    cin = synth.conv_states(1001, 1, H, D, taps).to(dev)
    cout = torch.empty_like(cin)
    csn = torch.empty((T // SNAP, 2, H, D, taps - 1), device=dev)

    def fe():
        K.kda_qk_frontend(rd["q"], rd["k"], wq, wk, cu, qo, ko, conv_in=cin, conv_out=cout,
                          snap_interval=SNAP, conv_snapshots=csn, chunk=C)
    ms_fe = time_calls(fe, steps, warmup, dev)
    cstate = 2 * H * D * (taps - 1) * 4
    b_fe = T * H * D * 2 * 4 + (2 + T // SNAP) * cstate
    x = synth.token_inputs(1002, n_seq, H, D, D, io="bf16")
    xd = {k: v.to(dev) for k, v in x.items()}
    rq = {k: v.to(dev) for k, v in synth.raw_qk(1002, n_seq, H, D, io="bf16").items()}
    pool = synth.states(1002, n_seq, H, D, D, std=0.1).to(dev)
    cpool = synth.conv_states(1002, n_seq, H, D, taps).to(dev)
    slots = torch.arange(n_seq, dtype=torch.int32, device=dev)
    o = torch.empty((n_seq, H, D), dtype=torch.bfloat16, device=dev)

    def dc():
        K.kda_decode_conv(rq["q"], rq["k"], xd["v"], xd["g"], xd["beta"], slots, pool, cpool, o,
                          wq, wk)
    ms_dc = time_calls(dc, steps, warmup, dev)
    b_dc = decode_bytes(n_seq) + n_seq * 2 * cstate
    st = K.kda_check_device_status()
    if st != 0:
        raise RuntimeError(f"front-end workloads: device status {K.kda_status_string(st)}")
    hbm = peaks["hbm_gbs"]
    return {
        "frontend_prefill": {"ms": round(ms_fe, 4), "value": T / (ms_fe * 1e-3), "unit": "tok/s",
                             "tokens": T, "algorithmic_bytes": b_fe,
                             "achieved_gbs": round(b_fe / (ms_fe * 1e-3) / 1e9, 1),
                             "hbm_frac": round(b_fe / (ms_fe * 1e-3) / 1e9 / hbm, 4),
                             "workload": "kda_qk_frontend, 8192 tokens x 64 heads, 4 taps, raw bf16 "
                                         "q/k in, normalised bf16 q/k out, conv snapshots /256"},
        "decode_conv": {"ms": round(ms_dc, 4), "value": n_seq * H / (ms_dc * 1e-3),
                        "unit": "state-steps/s", "algorithmic_bytes": b_dc,
                        "achieved_gbs": round(b_dc / (ms_dc * 1e-3) / 1e9, 1),
                        "hbm_frac": round(b_dc / (ms_dc * 1e-3) / 1e9 / hbm, 4),
                        "workload": "kda_decode_conv, 512 sequences x 64 heads, 4 taps, conv "
                                    "states updated in place with the fp32 states"},
    }


def time_calls(fn, steps, warmup, dev):
    """Average ms per call of fn() over `steps` calls after `warmup`, CUDA events."""
    stream = torch.cuda.current_stream(dev)
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize(dev)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        fn()
    b.record(stream)
    torch.cuda.synchronize(dev)
    return a.elapsed_time(b) / steps


def run_workload(args):
    """Single-workload timing lines (tiny fp32, ragged batch, 1M-token segments, the q/k
    front-end) used for the design notes and profiles; the default run is the serving step."""
    from hybrid_linear_attention_04_b200 import build as kbuild
    kbuild.build()
    from hybrid_linear_attention_04_b200 import kda as K
    dev = torch.device("cuda", 0)
    peaks = load_peaks()
    wl = synth.WORKLOADS
    out = {"impl": "ours", "workload": args.workload, "steps": args.steps, "warmup": args.warmup,
           "prefill_path": args.prefill_path}

    def workspace(xd, cu):
        if args.prefill_path != "split":
            return None
        n = K.kda_prefill_workspace_size(xd["q"], xd["v"], cu, C)
        return torch.empty(n, dtype=torch.uint8, device=dev) if n else None
    if args.workload == "tiny":
        r = bench_tiny(K, dev, args.steps, args.warmup)
        out.update({"unit": "us/call", "value": r["value"],
                    "graph_replay_us_per_call": r["graph_replay_us_per_call"],
                    "tokens": wl["tiny_fp32"]["T"]})
    elif args.workload == "ragged":
        c = wl["ragged_prefix_32"]
        plan = synth.ragged_plan(c["seed"], c["n_seq"], c["mu"], c["sigma"], c["lo"], c["hi"],
                                 c["prefix"], c["n_resume"], c["snap"])
        lens, start = plan["lens"], plan["start_pos"]
        cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
        T = int(cu[-1])
        x = synth.token_inputs(c["seed"], T, H, D, D, io="bf16")
        xd = {k: v.to(dev) for k, v in x.items()}
        del x
        s0 = synth.states(c["seed"], c["n_seq"], H, D, D, std=0.1).to(dev)
        o = torch.empty((T, H, D), dtype=torch.bfloat16, device=dev)
        so = torch.empty_like(s0)
        offs, _ = K.kda_snapshot_plan(cu, start, c["snap"])
        sn = torch.empty((int(offs[-1]), H, D, D), device=dev)
        ws = workspace(xd, cu)
        ms = time_calls(lambda: K.kda_prefill(xd["q"], xd["k"], xd["v"], xd["g"], xd["beta"], cu, o,
                                              state_out=so, state_in=s0, start_pos=start,
                                              snap_interval=c["snap"], snapshots=sn, chunk=C,
                                              workspace=ws),
                        args.steps, args.warmup, dev)
        byts = T * H * (3 * D * 2 + D * 2 + D * 4 + 4) + (int(offs[-1]) + 2 * c["n_seq"]) * H * D * D * 4
        out.update({"unit": "tok/s", "value": T / (ms * 1e-3), "ms": ms, "tokens": T,
                    "algorithmic_bytes": byts, "hbm_frac": byts / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"]})
    elif args.workload == "long":
        c = wl["long_1m"]
        seg, n_seg = c["segment"], c["T"] // c["segment"]
        # two distinct seeded segments alternate (identical work per call; the
        # host draws 2 of the 16 segments to keep set-up short)
        segs = []
        for i in range(2):
            x = synth.token_inputs(c["seed"], seg, H, D, D, io="bf16", t0=i * seg)
            segs.append({k: v.to(dev) for k, v in x.items()})
            del x
        o = torch.empty((seg, H, D), dtype=torch.bfloat16, device=dev)
        st = [torch.zeros((1, H, D, D), device=dev) for _ in range(2)]
        n_snap = seg // c["snap"]
        sn = torch.empty((n_snap, H, D, D), device=dev)
        cu = np.array([0, seg], dtype=np.int32)
        ws = workspace(segs[0], cu)

        def one_pass():
            for i in range(n_seg):
                xd = segs[i % 2]
                K.kda_prefill(xd["q"], xd["k"], xd["v"], xd["g"], xd["beta"], cu, o,
                              state_out=st[(i + 1) % 2], state_in=st[i % 2] if i else None,
                              start_pos=[i * seg], snap_interval=c["snap"], snapshots=sn, chunk=C,
                              workspace=ws)
        ms = time_calls(one_pass, max(1, args.steps // 5), 1, dev)
        T = c["T"]
        byts = T * H * (3 * D * 2 + D * 2 + D * 4 + 4) + (T // c["snap"] + 2 * n_seg) * H * D * D * 4
        out.update({"unit": "tok/s", "value": T / (ms * 1e-3), "ms": ms, "tokens": T,
                    "algorithmic_bytes": byts, "hbm_frac": byts / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"]})
    elif args.workload == "frontend":
        out.update(bench_frontend(K, dev, args.steps, args.warmup, peaks))
    st_ = K.kda_check_device_status()
    if st_ != 0:
        raise RuntimeError(K.kda_status_string(st_))
    print(json.dumps(out), flush=True)


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return None
    tok = args.ref_tokens
    for _ in range(args.warmup):
        cpu_baseline_prefill(tok, H)
    times, cores = [], 1
    for _ in range(args.steps):
        dt, cores = cpu_baseline_prefill(tok, H)
        times.append(dt)
    total = sum(times)
    val = args.steps * tok / total
    sample = f"fp64 token recurrence (the test oracle), first {tok} tokens x {H} heads of the " \
             f"prefill workload per step"
    result = {
        "impl": "reference", "metric": METRIC, "value": val, "unit": "tok/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * total / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "prefill 8192 tok x 64 heads (d=128, chunk 64, snapshots /256)"
                               " + decode/verify/commit 512 seq x 64 heads (drafts 1..8)",
                   "global_batch": 1 + N_SEQ, "seq_len": PREFILL_T, "parallelism": "cpu"},
        "cpu_baseline": {"value": val, "unit": "tok/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": val, "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(result), flush=True)
    return result


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-tokens", type=int, default=2048)
    ap.add_argument("--ref-tokens", type=int, default=512)
    ap.add_argument("--workload", choices=["serving", "tiny", "ragged", "long", "frontend"], default="serving")
    ap.add_argument("--prefill-tokens", type=int, default=PREFILL_T,
                    help="prefill length of the serving step (smaller only for profiler captures)")
    ap.add_argument("--decode-seqs", type=int, default=N_SEQ,
                    help="decode/verify sequences of the serving step (smaller only for profiler captures)")
    ap.add_argument("--serving-only", action="store_true",
                    help="time the serving step only (skip the tiny, ragged and 1M-token workloads)")
    ap.add_argument("--prefill-path", choices=["split", "fused"], default="split",
                    help="tensor-core prefill in two launches through a workspace (split) or in "
                         "one launch without one (fused)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)     # at least 3 untimed warm-up steps
    if args.impl == "reference":
        run_reference(args)
    elif args.workload != "serving":
        run_workload(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
