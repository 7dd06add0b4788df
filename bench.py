#!/usr/bin/env python
"""Benchmark of the TokenSwift verification hot path on B200.

One step = one pass of the whole per-step hot path on the LLaMA3.1-8B
100K-context workload (Hq=32, Hkv=8, D=128, n_ctx=102400, 40-node 3-ary
tree):
  1. ts_tree_verify_attn_root_scores over the full cache (the headline
     call; it also leaves the root node's scores over the context),
  2. ts_kv_select_from_scores: 64 sinks + top-4032 into the partial cache,
  3. the draft pass: ts_tree_verify_attn of a 4-node chain over that
     4096-row partial cache,
  4. ts_penalize_accept over fp32 logits [40, 128256], window 1024, on a
     second stream beside 2 and 3,
  5. ts_kv_commit_path: the accepted path's tree rows move to the end of
     the context (after 3 and 4).
With --select-score-pass, 1 and 2 are ts_tree_verify_attn and
ts_kv_importance_select (the select scores the context itself).
The metric counts tree-verify calls: each step holds exactly one.

Prints ONE JSON line (rank 0).  ``--impl reference`` times the fp64 CPU
oracle on a bounded sample of the same step instead.
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

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "tree-verify attn calls/s @100K ctx (LLaMA-8B GQA shape); % of HBM/tensor roofline"
UNIT = "calls/s"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default 1000; 3 for the reference arm, whose "
                         "steps take seconds each)")
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=50)
    ap.add_argument("--select-score-pass", action="store_true",
                    help="the select scores the context with its own pass over K instead "
                         "of taking the root node's scores from the verify attention")
    ap.add_argument("--no-sweep", action="store_true",
                    help="skip the 14B-shape roofline sweep (context x tree size)")
    ap.add_argument("--only", choices=["verify", "verify_plain", "select", "draft", "penalty",
                                       "penalty_sample", "commit"],
                    help="run one call of the step warmup + steps times, eagerly, and print "
                         "its mean device time (for profiler captures of a single kernel)")
    ap.add_argument("--breakdown", action="store_true",
                    help="device time of each call of the step alone (eager, CUDA events)")
    return ap.parse_args()


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def max_over_ranks(x: float, world: int, device) -> float:
    """The largest of every rank's x (a duration): the job is as slow as its
    slowest replica.  Single process: x itself."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(steps: int, world: int, ms_max: float) -> float:
    """Whole-job steps/s: every rank ran `steps` steps of its own problem
    (weak scaling) and the job took the slowest rank's ms_max."""
    return world * steps / (ms_max / 1e3)


def workload():
    from lossless_ultra_long_b200 import inputs as I
    return I.LLAMA8B_100K


def attn_bytes(hq, hkv, d, n_ctx, t, root_scores=True):
    """Algorithmic HBM bytes of one tree-verify call: K+V (context + tail, bf16),
    Q (bf16) and O (fp32), plus the root node's fp32 scores over the context
    when the call leaves them for the select."""
    return (4 * hkv * d * (n_ctx + t) + 2 * t * hq * d + 4 * t * hq * d +
            (4 * hq * n_ctx if root_scores else 0))


def attn_flops(hq, d, n_ctx, t):
    return 4 * hq * t * d * (n_ctx + t)


def measured_peaks(sustained=False):
    """(HBM GB/s, dense bf16 TFLOP/s, source): the machine's measured copy
    bandwidth and cuBLAS bf16 throughput (burst, or the seconds-long
    sustained figure for a kernel timed inside a long loop), else the
    fallback figures."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        tf = j.get("bf16_tflops_sustained") if sustained else None
        return float(j["hbm_gbs"]), float(tf or j["bf16_tflops"]), "measured"
    return 6650.0, 1400.0 if sustained else 1590.0, "fallback"


def attn_traffic_record():
    """DRAM bytes per launch of the attention call from a committed ncu capture,
    valid only while the kernel sources are unchanged since that capture."""
    p = os.path.join(ROOT, "profiles", "attn_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f)
    h = hashlib.sha256()
    for rel in rec.get("sources", []):
        path = os.path.join(ROOT, rel)
        if not os.path.exists(path):
            return None   # a source of the capture is gone: the record is stale
        with open(path, "rb") as f:
            h.update(f.read())
    if h.hexdigest() != rec.get("sources_sha256"):
        return None
    return float(rec["dram_bytes_per_call"])


def ngram_host_timing(L, n_tokens: int = 102400, steps: int = 2000, seed: int = 0) -> float:
    """Host microseconds per verification step of the n-gram reuse table:
    the step's accepted tokens (5: a depth-3 path and the bonus token) are
    counted and the new root's 8 most frequent continuations fetched, on a
    table that already holds the whole context (a Zipf(1.2) token stream
    over the workload's 128256-token vocabulary, n = 4)."""
    rng = np.random.default_rng(seed)
    text = np.minimum(rng.zipf(1.2, n_tokens + 5 * steps), 128255).astype(np.int32)
    tab = L.NgramTable(4, 1 << 18)   # fill limit 229376 n-grams
    tab.update(text[:n_tokens])
    t0 = time.perf_counter()
    for s in range(steps):
        end = n_tokens + 5 * (s + 1)
        tab.update(text[end - 8:end], 5)
        tab.topk(int(text[end - 1]), 8)
    return (time.perf_counter() - t0) / steps * 1e6


class ClockSampler:
    """SM clock and clock-event (throttle) reasons sampled during the timed
    region: NVML in a thread every 5 ms (read-only queries), else
    nvidia-smi at its fastest interval."""

    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40),
               ("sw_thermal_slowdown", 0x20), ("sw_power_cap", 0x4),
               ("hw_power_brake_slowdown", 0x80))

    def __init__(self, index: int, pci_bus_id: str | None = None):
        self.index = index
        self.pci = pci_bus_id
        self.samples, self.reason_bits, self.max_mhz = [], 0, None
        self.thread = self.proc = None
        import tempfile
        self.path = os.path.join(tempfile.gettempdir(), f"clocks_bench_{os.getpid()}.csv")

    def _nvml_loop(self, nv, h):
        import time
        while not self.stop:
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                self.reason_bits |= nv.nvmlDeviceGetCurrentClocksEventReasons(h)
            except Exception:
                pass
            time.sleep(0.005)

    def __enter__(self):
        self.stop = False
        try:
            import threading
            import pynvml as nv
            nv.nvmlInit()
            h = (nv.nvmlDeviceGetHandleByPciBusId(self.pci) if self.pci
                 else nv.nvmlDeviceGetHandleByIndex(self.index))
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
            self.thread = threading.Thread(target=self._nvml_loop, args=(nv, h), daemon=True)
            self.thread.start()
            return self
        except Exception:
            self.thread = None
        os.makedirs(os.path.dirname(self.path), exist_ok=True)
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={q}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=self.fh, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.stop = True
        if self.thread is not None:
            self.thread.join(timeout=2)
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.fh.close()

    def summary(self):
        if self.thread is not None:
            sm = self.samples
            reasons = sorted(n for n, bit in self.REASONS if self.reason_bits & bit)
            return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": self.max_mhz,
                    "samples": len(sm), "source": "nvml", "reasons": reasons}
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax = float(parts[2])
                except ValueError:
                    continue
                for name, val in zip(names, parts[5:9]):
                    if val.lower() == "active":
                        reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "samples": len(sm), "source": "nvidia-smi", "reasons": sorted(reasons)}


# --------------------------------------------------------------------- ours
class Step:
    """Device-resident buffers and the four ABI calls of one verification step."""

    def __init__(self, torch, L, I, w, dev, fused=True, want_scores=False):
        from_bits = lambda b: torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).view(
            torch.bfloat16).to(dev)
        self.torch, self.L, self.w = torch, L, w
        self.parent = w.parent()
        self.draft_parent = I.chain_tree(w.draft_tree)
        q = I.gen_q(w)
        k, v = I.gen_kv(w)
        self.q = from_bits(q)
        self.k, self.v = from_bits(k), from_bits(v)
        del k, v
        lg = I.gen_logits(w)
        tokens, lg = I.gen_tree_tokens(w, self.parent, lg)
        self.logits = torch.from_numpy(lg).to(dev)
        self.window = torch.from_numpy(I.gen_window(w)).to(dev)
        self.tokens = torch.from_numpy(tokens).to(dev)
        hq, hkv, d = w.n_heads_q, w.n_heads_kv, w.head_dim
        self.n_keep = w.n_sink + w.budget
        cap = self.n_keep + w.draft_tree
        self.kp = torch.zeros((hkv, cap, d), dtype=torch.bfloat16, device=dev)
        self.vp = torch.zeros_like(self.kp)
        # the draft chain's own K/V rows sit after the kept rows
        dk = I.gen_q(w.with_(seed=w.seed + 100), n_nodes=w.draft_tree)   # any seeded bf16 rows
        self.kp[:, self.n_keep:] = from_bits(dk[:, :hkv, :].transpose(1, 0, 2))
        self.vp[:, self.n_keep:] = from_bits(dk[:, hkv:2 * hkv, :].transpose(1, 0, 2))
        self.dq = from_bits(I.gen_draft_q(w))
        self.idx = torch.empty((hkv, self.n_keep), dtype=torch.int32, device=dev)
        self.out = torch.empty((w.n_tree, hq, d), dtype=torch.float32, device=dev)
        self.dout = torch.empty((w.draft_tree, hq, d), dtype=torch.float32, device=dev)
        self.accept = torch.empty(2 + w.n_tree, dtype=torch.int32, device=dev)
        self.argmax = torch.empty(w.n_tree, dtype=torch.int32, device=dev)
        self.ws_attn = L.new_workspace(L.tree_verify_attn_workspace_size(hq, hkv, d, w.n_ctx,
                                                                         w.n_tree), dev)
        self.ws_draft = L.new_workspace(L.tree_verify_attn_workspace_size(
            hq, hkv, d, self.n_keep, w.draft_tree), dev)
        # the root node's base-2 scores, left by the verify attention for the
        # select (or, unfused, computed by the select's own score pass)
        self.fused = fused
        if fused:
            self.rs = torch.empty((hq, w.n_ctx), dtype=torch.float32, device=dev)
            self.ws_sel = L.new_workspace(L.kv_select_from_scores_workspace_size(hq, hkv, w.n_ctx),
                                          dev)
        else:
            self.rs = None
            self.ws_sel = L.new_workspace(
                L.kv_importance_select_workspace_size(hq, hkv, d, w.n_ctx), dev)
        self.ws_pen = L.new_workspace(L.penalize_accept_workspace_size(w.n_tree, w.vocab), dev)
        self.ws_commit = L.new_workspace(256, dev)
        # the importance scores the select ranks by, when a caller wants to see them
        self.scores = (torch.empty((hkv, w.n_ctx), dtype=torch.float32, device=dev)
                       if want_scores else None)
        self.side = torch.cuda.Stream(device=dev)

    def attn(self, root_scores=True):
        self.L.tree_verify_attn(self.q, self.k, self.v, self.w.n_ctx, self.parent, out=self.out,
                                workspace=self.ws_attn,
                                root_scores_out=self.rs if root_scores else None)

    def select(self):
        w, L = self.w, self.L
        if self.fused:
            L.kv_select_from_scores(self.rs, self.k, self.v, w.n_ctx, w.n_sink, w.budget,
                                    k_partial=self.kp, v_partial=self.vp, idx_out=self.idx,
                                    scores_out=self.scores, workspace=self.ws_sel)
        else:
            L.kv_importance_select(self.q[0], self.k, self.v, w.n_ctx, w.n_sink, w.budget,
                                   k_partial=self.kp, v_partial=self.vp, idx_out=self.idx,
                                   scores_out=self.scores, workspace=self.ws_sel)

    def penalty(self):
        w = self.w
        self.L.penalize_accept(self.logits, self.window, w.penalty, self.parent, self.tokens,
                               argmax_out=self.argmax, accept_out=self.accept,
                               workspace=self.ws_pen)

    def penalty_sample(self, temperature=0.8):
        """The penalty call with temperature acceptance (the Gumbel-max
        draw); the noise is drawn once, on the device, on first use."""
        w = self.w
        if getattr(self, "gumbel", None) is None:
            gen = self.torch.Generator(device=self.logits.device)
            gen.manual_seed(w.seed)
            u = self.torch.rand(self.logits.shape, generator=gen, device=self.logits.device,
                                dtype=self.torch.float64).clamp_min_(2.0 ** -1022)
            self.gumbel = (-(-u.log()).log()).float()
            del u
        self.L.penalize_sample_accept(self.logits, self.gumbel, temperature, self.window,
                                      w.penalty, self.parent, self.tokens,
                                      target_out=self.argmax, accept_out=self.accept,
                                      workspace=self.ws_pen)

    def draft(self):
        self.L.tree_verify_attn(self.dq, self.kp, self.vp, self.n_keep, self.draft_parent,
                                out=self.dout, workspace=self.ws_draft)

    def commit(self):
        """The accepted path's tree rows become the context's next rows."""
        w = self.w
        self.L.kv_commit_path(self.k, self.v, w.n_ctx, w.n_tree, self.accept,
                              workspace=self.ws_commit)

    def rest(self):
        """Select, then the draft pass over the partial cache it builds; the
        penalty/accept call depends on neither and runs beside them on a
        second stream; the commit of the accepted path follows both."""
        torch = self.torch
        main = torch.cuda.current_stream()
        self.side.wait_stream(main)   # fork: the side stream depends on what came before
        self.select()
        # enqueued after the select so that its kernels start first and the
        # penalty CTAs fill the SMs they leave
        with torch.cuda.stream(self.side):
            self.penalty()
        self.draft()
        main.wait_stream(self.side)
        self.commit()

    def step(self):
        self.attn()
        self.rest()


def run_ours(args):
    import torch
    import torch.distributed as dist
    import lossless_ultra_long_b200 as L
    from lossless_ultra_long_b200 import inputs as I

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    L.library()
    w = workload()
    st = Step(torch, L, I, w, dev, fused=not args.select_score_pass)
    stream = torch.cuda.Stream(device=dev)

    # warm-up eagerly (sets kernel attributes), then capture the step as one
    # CUDA graph (no event nodes inside it: two event records inside a step
    # graph measured about 5 us per step on a B200 and added 3-4 us to the
    # interval they bracket)
    with torch.cuda.stream(stream):
        for _ in range(max(args.warmup, 3)):
            st.step()
    stream.synchronize()
    g_step = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_step, stream=stream, capture_error_mode="thread_local"):
        st.attn()
        st.rest()
    # the verify call alone: ten back-to-back calls per graph
    kAttnPerGraph = 10
    g_attn = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_attn, stream=stream, capture_error_mode="thread_local"):
        for _ in range(kAttnPerGraph):
            st.attn()
    with torch.cuda.stream(stream):
        for _ in range(max(args.warmup, 3)):
            g_step.replay()
        g_attn.replay()
    stream.synchronize()

    launches_per_step = None
    c0 = L.kernel_launch_count()
    with torch.cuda.stream(stream):
        st.step()
    stream.synchronize()
    launches_per_step = L.kernel_launch_count() - c0

    K = args.steps
    attn_reps = max(5, min(30, K // kAttnPerGraph))
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    props = torch.cuda.get_device_properties(dev)
    pci = None
    if hasattr(props, "pci_bus_id"):
        pci = "%08X:%02X:%02X.0" % (getattr(props, "pci_domain_id", 0), props.pci_bus_id,
                                    getattr(props, "pci_device_id", 0))
    with ClockSampler(local, pci) as clk:
        # the timed steps
        with torch.cuda.stream(stream):
            t0.record(stream)
            for i in range(K):
                g_step.replay()
            t1.record(stream)
        torch.cuda.synchronize()
        # right after, under the same clock sampling: the verify call's
        # device time, from events on its stream around graphs of
        # back-to-back calls (inputs 420 MB, far above L2)
        with torch.cuda.stream(stream):
            a0.record(stream)
            for i in range(attn_reps):
                g_attn.replay()
            a1.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms_total = t0.elapsed_time(t1)
    ms_max = max_over_ranks(ms_total, world, dev)
    attn_ms = max_over_ranks(a0.elapsed_time(a1) / (attn_reps * kAttnPerGraph), world, dev)

    # end to end through the public API: per step, pinned host inputs are
    # copied in, the four calls run, and the results are read back
    e2e = run_e2e(torch, L, st, w, dev, stream, args.e2e_steps)
    e2e_ms = max_over_ranks(e2e["ms_per_step"], world, dev)

    out = None
    if rank == 0:
        hbm, tflops, src = measured_peaks(sustained=True)
        attn_avg_s = attn_ms / 1e3
        # the call's algorithmic bytes (K + V + Q + O); the fused call also
        # writes the root node's scores, counted separately
        byts = attn_bytes(w.n_heads_q, w.n_heads_kv, w.head_dim, w.n_ctx, w.n_tree,
                          root_scores=False)
        score_bytes = (attn_bytes(w.n_heads_q, w.n_heads_kv, w.head_dim, w.n_ctx, w.n_tree,
                                  root_scores=True) - byts) if st.fused else 0
        flops = attn_flops(w.n_heads_q, w.head_dim, w.n_ctx, w.n_tree)
        achieved = byts / attn_avg_s / 1e9
        value = job_throughput(K, world, ms_max)
        e2e_value = job_throughput(1, world, e2e_ms)
        out = {
            "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
            "steps": K, "warmup": args.warmup, "ms_per_step": round(ms_max / K, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": w.name, "n_heads_q": w.n_heads_q, "n_heads_kv": w.n_heads_kv,
                       "head_dim": w.head_dim, "n_ctx": w.n_ctx, "n_tree": w.n_tree,
                       "tree": "3-ary BFS depth 3", "step": ("verify attn (leaving the root's scores) + importance "
                                "select from them" if st.fused else "verify attn + importance "
                                "select with its own score pass") + " (64+4032) + 4-node draft attn over the partial cache + penalty/accept "
                       "(V=128256, W=1024) + commit of the accepted path; penalty/accept on a second stream beside the "
                       "select and draft pass", "l2": "inputs larger than L2 (420 MB KV per step)",
                       "parallelism": f"replicas x{world}", "graphs": True,
                       "attn_timing": "events around %d graphs of %d back-to-back verify calls, "
                                      "right after the timed steps" % (attn_reps, kAttnPerGraph)},
            "attn_call_us": round(attn_avg_s * 1e6, 2),
            "attn_only_calls_per_s": round(1.0 / attn_avg_s, 1),
            "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm,
                         "unit": "GB/s", "frac": round(achieved / hbm, 4),
                         "peak_source": src, "traffic": attn_traffic_record(),
                         "algorithmic_bytes": byts, "root_score_bytes": score_bytes,
                         "frac_with_root_scores": round((byts + score_bytes) / attn_avg_s /
                                                        1e9 / hbm, 4),
                         "tensor_frac": round(flops / attn_avg_s / 1e12 / tflops, 4),
                         "tensor_peak_tflops": tflops},
            "e2e": {"value": round(e2e_value, 2), "unit": UNIT,
                    "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"]},
            "gpu_launches": int(launches_per_step * K),
            "clocks": clk.summary(),
        }
        try:
            out["ngram_host_us_per_step"] = round(ngram_host_timing(L), 2)
        except Exception as e:   # host-side extra: never costs the GPU line
            out["ngram_host_us_per_step"] = None
            out["ngram_host_error"] = str(e)[:200]
        if not args.no_sweep:
            hbm_b, tf_b, _ = measured_peaks(sustained=False)
            out["sweep"] = sweep_14b(torch, L, I, dev, hbm_b, tf_b)
        if not args.no_cpu_baseline:
            out["cpu_baseline"] = cpu_baseline(w)
    if world > 1:
        dist.barrier()
        del g_step, g_attn
        dist.destroy_process_group()
    return out


def _setup_single(args):
    """Device, library and the step's buffers for the single-call modes."""
    import torch
    import lossless_ultra_long_b200 as L
    from lossless_ultra_long_b200 import inputs as I
    _, _, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    L.library()
    st = Step(torch, L, I, workload(), dev, fused=not args.select_score_pass)
    return torch, L, st


def _call_of(st, name):
    return {"verify": lambda: st.attn(True), "verify_plain": lambda: st.attn(False),
            "select": st.select, "draft": st.draft, "penalty": st.penalty,
            "penalty_sample": st.penalty_sample, "commit": st.commit}[name]


def _prepare(st, name):
    """Inputs a call reads that an earlier call of the step produces."""
    if name in ("select", "draft"):
        st.attn(True)
    if name == "draft":
        st.select()
    if name == "commit":
        st.penalty()


def _time_call(torch, fn, warmup, steps):
    """Mean device time (us) of fn over `steps` back-to-back calls after
    `warmup` calls, CUDA events on the current stream."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) * 1e3 / max(steps, 1)


def run_only(args):
    """One call of the step, run warmup + steps times eagerly (a short,
    self-contained program for profiler captures of one kernel)."""
    torch, L, st = _setup_single(args)
    _prepare(st, args.only)
    fn = _call_of(st, args.only)
    us = _time_call(torch, fn, args.warmup, args.steps)
    return {"mode": "only", "call": args.only, "workload": st.w.name, "steps": args.steps,
            "warmup": args.warmup, "us_per_call": round(us, 2),
            "launches": L.kernel_launch_count()}


def _time_call_graph(torch, fn, warmup, steps, per_graph=10):
    """Mean device time (us) of fn, replayed from a CUDA graph that holds
    per_graph back-to-back calls (no host launch cost between calls)."""
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        for _ in range(max(warmup, 3)):
            fn()
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream, capture_error_mode="thread_local"):
        for _ in range(per_graph):
            fn()
    reps = max(1, steps // per_graph)
    with torch.cuda.stream(stream):
        g.replay()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            g.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) * 1e3 / (reps * per_graph)


def run_breakdown(args):
    """Device time of each call of the step alone, back to back inside a
    CUDA graph (the verify call reads 420 MB per call, so it runs from HBM;
    the smaller calls re-read inputs that may sit in L2)."""
    torch, L, st = _setup_single(args)
    w = st.w
    st.attn(True)
    st.select()
    st.penalty()
    out = {"mode": "breakdown", "workload": w.name, "timing": "CUDA graph of 10 calls"}
    st.penalty_sample()   # draws the noise outside the timed graphs
    for name in ("verify", "verify_plain", "select", "draft", "penalty", "penalty_sample",
                 "commit"):
        out[name + "_us"] = round(_time_call_graph(torch, _call_of(st, name), args.warmup,
                                                   max(args.steps, 10)), 2)
    return out


def sweep_14b(torch, L, I, dev, hbm, tflops, warmup=10, calls=50):
    """The 14B GQA roofline sweep: Hq 40, Hkv 8, D 128, contexts 4K-131K and
    trees of 4 (a chain), 13 and 40 nodes.  Per point: the verify call's mean
    device time over back-to-back calls, replayed from a CUDA graph (so that
    host launch cost does not time the short calls), that rotate over enough
    copies of the KV cache that each call reads from HBM (3 x L2 at least),
    its algorithmic bytes and flops, achieved GB/s and TFLOP/s and their
    fractions of the measured peaks.  Inputs: seeded N(0, 1) bf16 drawn on
    the device."""
    l2 = 126 * 2 ** 20
    points = []
    gen = torch.Generator(device=dev)
    for n_ctx in I.SWEEP_CTX:
        t_max = max(I.SWEEP_TREE)
        hkv, hq, d = 8, 40, 128
        kv_bytes = 2 * hkv * (n_ctx + t_max) * d * 2
        n_sets = max(1, min(24, -(-3 * l2 // kv_bytes)))
        gen.manual_seed(4000 + n_ctx)
        sets = []
        for _ in range(n_sets):
            k = torch.randn((hkv, n_ctx + t_max, d), generator=gen, device=dev).to(torch.bfloat16)
            v = torch.randn((hkv, n_ctx + t_max, d), generator=gen, device=dev).to(torch.bfloat16)
            sets.append((k, v))
        for t in I.SWEEP_TREE:
            w = I.sweep14b(n_ctx, t)
            parent = w.parent()
            q = torch.randn((t, hq, d), generator=gen, device=dev).to(torch.bfloat16)
            out = torch.empty((t, hq, d), dtype=torch.float32, device=dev)
            ws = L.new_workspace(L.tree_verify_attn_workspace_size(hq, hkv, d, n_ctx, t), dev)
            it = [0]

            def call():
                k, v = sets[it[0] % n_sets]
                it[0] += 1
                L.tree_verify_attn(q, k, v, n_ctx, parent, out=out, workspace=ws)

            # one graph of a whole number of rotations, at least 10 calls
            per_graph = n_sets * max(1, -(-10 // n_sets))
            us = _time_call_graph(torch, call, warmup, calls, per_graph=per_graph)
            byts = attn_bytes(hq, hkv, d, n_ctx, t, root_scores=False)
            flops = attn_flops(hq, d, n_ctx, t)
            gbs = byts / (us * 1e-6) / 1e9
            tfs = flops / (us * 1e-6) / 1e12
            points.append({"n_ctx": n_ctx, "n_tree": t, "us": round(us, 2),
                           "calls_per_s": round(1e6 / us, 1), "bytes": byts, "flops": flops,
                           "gbs": round(gbs, 1), "hbm_frac": round(gbs / hbm, 4),
                           "tflops": round(tfs, 1), "tensor_frac": round(tfs / tflops, 4)})
        del sets
        torch.cuda.empty_cache()
    return {"workload": "qwen14b_gqa40x8_d128", "kv_sets_rotated": "ceil(3 x L2 / KV bytes), "
            "at most 24", "calls_per_point": calls, "timing": "CUDA graph of whole rotations, "
            "events around its replays", "points": points}


def run_e2e(torch, L, st, w, dev, stream, steps):
    """The same step through the Python API with host buffers: H2D of the
    step's new inputs (queries, the tree's own K/V rows, logits, window,
    tree tokens, draft queries) from pinned memory, the calls, D2H of the
    results (outputs, accept, kept indices), and a host wait for them every
    step.  The penalty/accept inputs are uploaded on the stream that call
    runs on, overlapping the verify attention.  After an eager warm-up the
    calls and copies are captured once as a CUDA graph, replayed once per
    step."""
    hq, hkv, d, t = w.n_heads_q, w.n_heads_kv, w.head_dim, w.n_tree
    pin = lambda x: x.cpu().pin_memory()
    h_q, h_dq = pin(st.q), pin(st.dq)
    h_kt = pin(st.k[:, w.n_ctx:w.n_ctx + t])
    h_vt = pin(st.v[:, w.n_ctx:w.n_ctx + t])
    h_lg, h_win, h_tok = pin(st.logits), pin(st.window), pin(st.tokens)
    o_out = torch.empty_like(st.out, device="cpu").pin_memory()
    o_dout = torch.empty_like(st.dout, device="cpu").pin_memory()
    o_acc = torch.empty_like(st.accept, device="cpu").pin_memory()
    o_idx = torch.empty_like(st.idx, device="cpu").pin_memory()
    h2d = sum(x.numel() * x.element_size() for x in (h_q, h_dq, h_kt, h_vt, h_lg, h_win, h_tok))
    d2h = sum(x.numel() * x.element_size() for x in (o_out, o_dout, o_acc, o_idx))

    def one():
        # the penalty/accept call's inputs (the 20 MB of logits above all) go
        # up on the side stream it runs on, so that their copy overlaps the
        # verify attention, which does not need them; the attention's and
        # the draft pass's inputs go up on the main stream
        with torch.cuda.stream(st.side):
            st.logits.copy_(h_lg, non_blocking=True)
            st.window.copy_(h_win, non_blocking=True)
            st.tokens.copy_(h_tok, non_blocking=True)
        st.q.copy_(h_q, non_blocking=True)
        st.dq.copy_(h_dq, non_blocking=True)
        st.k[:, w.n_ctx:w.n_ctx + t].copy_(h_kt, non_blocking=True)
        st.v[:, w.n_ctx:w.n_ctx + t].copy_(h_vt, non_blocking=True)
        st.step()
        o_out.copy_(st.out, non_blocking=True)
        o_dout.copy_(st.dout, non_blocking=True)
        o_acc.copy_(st.accept, non_blocking=True)
        o_idx.copy_(st.idx, non_blocking=True)
        stream.synchronize()

    with torch.cuda.stream(stream):
        for _ in range(3):
            one()
    # the same calls and copies captured once as a CUDA graph: a step is then
    # one launch, the host still waiting for each step's results
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream, capture_error_mode="thread_local"):
        with torch.cuda.stream(st.side):
            st.logits.copy_(h_lg, non_blocking=True)
            st.window.copy_(h_win, non_blocking=True)
            st.tokens.copy_(h_tok, non_blocking=True)
        st.q.copy_(h_q, non_blocking=True)
        st.dq.copy_(h_dq, non_blocking=True)
        st.k[:, w.n_ctx:w.n_ctx + t].copy_(h_kt, non_blocking=True)
        st.v[:, w.n_ctx:w.n_ctx + t].copy_(h_vt, non_blocking=True)
        st.step()
        o_out.copy_(st.out, non_blocking=True)
        o_dout.copy_(st.dout, non_blocking=True)
        o_acc.copy_(st.accept, non_blocking=True)
        o_idx.copy_(st.idx, non_blocking=True)
    with torch.cuda.stream(stream):
        for _ in range(3):
            g.replay()
            stream.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            g.replay()
            stream.synchronize()   # the host reads each step's results
        e1.record(stream)
    torch.cuda.synchronize()
    return {"ms_per_step": e0.elapsed_time(e1) / steps, "h2d": h2d, "d2h": d2h}


# ----------------------------------------------------------- the oracle
class OracleSample:
    """The fp64 oracle on a bounded sample of one step, scaled to a full step.

    attn_rows of the T*Hq verify-attention rows, the importance select of
    every KV head over the first sel_positions context positions, draft_rows
    of the draft pass's rows, pen_nodes of the tree nodes' penalty/argmax,
    and the acceptance walk; each part's time is scaled by the share it
    sampled.  The oracle spreads rows, heads and nodes over the host's
    threads, so every sampled part keeps all of them busy (at least one row
    or node per thread, all heads) and the scaling does not charge idle
    threads to the full step."""

    def __init__(self, w, attn_rows, sel_positions, draft_rows, pen_nodes):
        import oracle
        from lossless_ultra_long_b200 import inputs as I
        oracle.build()
        self.o, self.w = oracle, w
        self.attn_rows, self.sel_positions = attn_rows, min(sel_positions, w.n_ctx)
        self.draft_rows, self.pen_nodes = draft_rows, pen_nodes
        self.q = I.gen_q(w)
        self.k, self.v = I.gen_kv(w)
        self.parent = w.parent()
        self.n_keep = w.n_sink + w.budget
        self.dq = I.gen_draft_q(w)
        self.kp = np.ascontiguousarray(self.k[:, : self.n_keep + w.draft_tree])
        self.vp = np.ascontiguousarray(self.v[:, : self.n_keep + w.draft_tree])
        self.dparent = I.chain_tree(w.draft_tree)
        lg = I.gen_logits(w)
        self.tokens, self.lg = I.gen_tree_tokens(w, self.parent, lg)
        self.win = I.gen_window(w)
        self.rng = np.random.default_rng(0)
        self.sample = (f"{attn_rows} of {w.n_tree * w.n_heads_q} verify-attention rows; "
                       f"importance select of all {w.n_heads_kv} KV heads over "
                       f"{self.sel_positions} of {w.n_ctx} positions; {draft_rows} of "
                       f"{w.draft_tree * w.n_heads_q} draft-pass rows; penalty/argmax of "
                       f"{pen_nodes} of {w.n_tree} nodes; acceptance and commit; scaled to one step")

    def seconds_per_step(self):
        o, w = self.o, self.w
        rows_total = w.n_tree * w.n_heads_q
        sel = self.rng.choice(rows_total, size=self.attn_rows, replace=False)
        t0 = time.perf_counter()
        o.tree_verify_attn_rows(self.q, self.k, self.v, w.n_ctx, self.parent,
                                (sel // w.n_heads_q).astype(np.int32),
                                (sel % w.n_heads_q).astype(np.int32))
        t_attn = (time.perf_counter() - t0) * rows_total / self.attn_rows
        g, n = w.group, self.sel_positions
        t0 = time.perf_counter()
        sc = o.importance_scores(self.q[0], self.k, n, w.n_heads_q)
        idx = o.select_topk(sc, w.n_sink, w.budget)
        o.gather_rows(self.k, idx)
        o.gather_rows(self.v, idx)
        t_sel = (time.perf_counter() - t0) * w.n_ctx / n
        drows = w.draft_tree * w.n_heads_q
        dsel = self.rng.choice(drows, size=self.draft_rows, replace=False)
        t0 = time.perf_counter()
        o.tree_verify_attn_rows(self.dq, self.kp, self.vp, self.n_keep, self.dparent,
                                (dsel // w.n_heads_q).astype(np.int32),
                                (dsel % w.n_heads_q).astype(np.int32))
        t_draft = (time.perf_counter() - t0) * drows / self.draft_rows
        t0 = time.perf_counter()
        am = o.penalize_argmax(self.lg[: self.pen_nodes], self.win, w.penalty)
        t_pen = (time.perf_counter() - t0) * w.n_tree / self.pen_nodes
        am_full = np.resize(am, w.n_tree).astype(np.int32)
        t0 = time.perf_counter()
        acc = o.accept_longest(self.parent, self.tokens, am_full)
        # the commit touches the tree-tail rows only
        lo, hi = w.n_ctx, w.n_ctx + w.n_tree
        o.kv_commit_path(self.k[:, lo:hi], 0, w.n_tree, acc)
        o.kv_commit_path(self.v[:, lo:hi], 0, w.n_tree, acc)
        t_acc = time.perf_counter() - t0
        return t_attn + t_sel + t_draft + t_pen + t_acc


def oracle_threads():
    return int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def cpu_baseline(w):
    """About 10-30 s of oracle work on the host cores (rank 0, N = 1 leg):
    a sampled step on all cores, and a smaller sample on one thread."""
    import oracle
    thr = oracle_threads()
    smp = OracleSample(w, attn_rows=160, sel_positions=w.n_ctx, draft_rows=128, pen_nodes=40)
    per_step = smp.seconds_per_step()
    one = OracleSample(w, attn_rows=16, sel_positions=8192, draft_rows=16, pen_nodes=8)
    oracle.set_num_threads(1)
    try:
        per_step_1 = one.seconds_per_step()
    finally:
        oracle.set_num_threads(thr)
    return {"value": round(1.0 / per_step, 6), "unit": UNIT, "cores": thr,
            "kind": "oracle", "sample": smp.sample, "seconds_per_step": round(per_step, 3),
            "cpu_model": cpu_model(),
            "one_thread": {"value": round(1.0 / per_step_1, 6), "unit": UNIT, "cores": 1,
                           "sample": one.sample, "seconds_per_step": round(per_step_1, 3)}}


def run_reference(args):
    """The oracle timed on the host cores, whole steps: every verify row,
    the importance select over the whole context with the gather, every
    draft-pass row, the penalty/argmax of every node and the acceptance --
    no sampling and no scaling.  Rank 0 only."""
    rank, world, _ = dist_env()
    if rank != 0:
        return None
    w = workload()
    K = max(1, args.steps)
    thr = oracle_threads()
    smp = OracleSample(w, attn_rows=w.n_tree * w.n_heads_q, sel_positions=w.n_ctx,
                       draft_rows=w.draft_tree * w.n_heads_q, pen_nodes=w.n_tree)
    for _ in range(min(args.warmup, 1)):
        smp.seconds_per_step()
    secs = [smp.seconds_per_step() for _ in range(K)]
    per_step = statistics.mean(secs)
    val = round(1.0 / per_step, 6)
    return {"metric": METRIC, "value": val, "unit": UNIT, "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": round(per_step * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": w.name, "n_heads_q": w.n_heads_q, "n_heads_kv": w.n_heads_kv,
                       "head_dim": w.head_dim, "n_ctx": w.n_ctx, "n_tree": w.n_tree},
            "cpu_baseline": {"value": val, "unit": UNIT, "cores": thr, "kind": "oracle",
                             "sample": "whole steps: " + smp.sample.replace(
                                 "; scaled to one step", ""),
                             "cpu_model": cpu_model(), "warmup_steps": min(args.warmup, 1)},
            "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    args = parse()
    if args.steps is None:
        args.steps = 3 if args.impl == "reference" else 1000
    if args.impl == "reference":
        out = run_reference(args)
    elif args.only:
        out = run_only(args)
    elif args.breakdown:
        out = run_breakdown(args)
    else:
        out = run_ours(args)
    if out is not None:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
