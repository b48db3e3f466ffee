"""Benchmark of the DSA prefill hot path: lightning indexer -> per-row top-k -> sparse
absorbed MLA, one layer at T = 65536 with top-2048 (16 indexer heads x 64, 16 query heads,
576-dim latent), on synthetic seeded inputs.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Prints one JSON line (rank 0).  With N > 1 (launched by torchrun) every rank runs its own
independent sequence (weak scaling, no data-path collective); the time is the max over
ranks.  ``--impl reference`` times the CPU oracle on a bounded sample of query rows.
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


ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

METRIC = "DSA prefill tokens/sec at T=64K, top-2048 (indexer+top-k+sparse MLA); % roofline"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--T", type=int, default=65536, help="sequence length (default 65536)")
    ap.add_argument("--topk", type=int, default=2048)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-decode", action="store_true",
                    help="skip the decode workload that the default prefill line carries as "
                         "its nested 'decode' object")
    ap.add_argument("--no-rows", action="store_true",
                    help="N>1: skip the row-sharded strong-scaling measurement that the "
                         "default line carries as its nested 'strong_scaling' object")
    ap.add_argument("--workload", choices=["prefill", "decode", "stack", "varlen"],
                    default="prefill",
                    help="prefill: the T=65536 headline; decode: 64 sequences x 32768 paged "
                         "tokens; stack: the 27-layer FSS x 9 IndexCache stack at T=16384; "
                         "varlen: 16 packed prompts of 512..8192 tokens in one batch")
    ap.add_argument("--shard", choices=["sequences", "rows"], default="sequences",
                    help="N>1: sequences = one sequence per rank (weak scaling); rows = the "
                         "query rows of one T-token prefill split over the ranks (strong "
                         "scaling, one all-gather of keys and latent rows per step)")
    ap.add_argument("--kv-dtype", choices=["bf16", "fp8"], default="bf16",
                    help="latent cache: bf16, or E4M3 codes times one fp32 scale")
    ap.add_argument("--window-rows", type=int, default=0,
                    help="query rows per indexer/top-k window (0 = the library default)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="target CPU time of the oracle baseline sample")
    return ap.parse_args(argv)


# ----------------------------------------------------------------------------------
# workload
# ----------------------------------------------------------------------------------
def make_inputs(T, k, seed, kv_dtype="bf16"):
    from sparse_attention_17_b200 import inputs as G
    if kv_dtype == "fp8":
        return G.mla_prefill_gauss_fp8(T=T, seed=seed, k=k)
    return G.mla_prefill_gauss(T=T, seed=seed, k=k)


def algorithmic_work(T, k, kv_bytes=2):
    """FLOPs and bytes of one prefill step, counted from the definitions (kv_bytes: bytes
    per latent element, 2 for bf16, 1 for E4M3 codes)."""
    causal = T * (T + 1) // 2                       # (t, s) pairs with s <= t
    sel = sum(min(t + 1, k) for t in range(T))      # selected keys over all queries
    return {
        "indexer_flop": 2 * 16 * 64 * causal,       # 16 heads x 64-dim dot per pair
        "mla_flop": 2 * 16 * (576 + 512) * sel,     # QK (576) + PV (512) per head per key
        "mla_gather_bytes": 576 * kv_bytes * sel,   # one 576-element latent row per key
        "topk_read_bytes": 4 * causal,              # fp32 scores read once per pair
        "hbm_bytes": (T * 16 * 64 * 2 + T * 64 * 2 + T * 16 * 4 + T * 16 * 576 * 2
                      + T * 576 * kv_bytes + T * 16 * 512 * 2 + 2 * T * k * 4),
    }


def shard_plan(rank, world, T, k):
    """Weak scaling over independent sequences: rank r prefills its own length-T sequence
    (inputs seeded r); nothing crosses ranks on the data path."""
    if not 0 <= rank < world:
        raise ValueError("rank out of range")
    return {"seed": rank, "T": T, "topk": k, "tokens": T}


def max_over_ranks(x, device=None):
    """Max of a per-rank float over the process group (identity without one)."""
    import torch
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_tokens_per_s(tokens_per_rank, world, ms_per_step):
    """Whole-job throughput: all ranks' tokens over the slowest rank's step time."""
    return world * tokens_per_rank / (ms_per_step / 1e3)


# Random 1152-byte latent rows gathered from an L2-resident cache into shared memory, all
# 148 SMs, no compute: the best rate measured on this B200 (16-byte cp.async from 8 warps
# per SM, 38 B/clk/SM at 1965 MHz).  The sparse-MLA prefill reads every selected row this
# way, so this is its gather ceiling next to the tensor-core roofline.
L2_GATHER_PEAK_TBS = 10.8
L2_GATHER_PEAK_SOURCE = ("measured gather micro-benchmark: random 1152 B rows of a 75 MB "
                         "L2-resident buffer into shared memory, 148 SMs, 16-byte cp.async")


def choose_tensor_peak(peaks, clocks):
    """The burst bf16 peak when the timed region ran at the maximum SM clock with no power
    cap (a kernel timed under burst conditions), else the sustained one."""
    burst, sust = peaks.get("bf16_tflops"), peaks.get("bf16_tflops_sustained")
    mhz, mx = clocks.get("sm_mhz"), clocks.get("sm_max_mhz")
    at_max = mhz is not None and mx and mhz >= 0.97 * mx
    if burst and (at_max and "sw_power_cap" not in clocks.get("reasons", []) or not sust):
        return burst, (f"burst (timed region at {mhz:.0f} of {mx:.0f} MHz, no power cap)"
                       if at_max else "burst")
    return sust, (f"sustained (timed region at {mhz} of {mx} MHz or under a power cap)")


def load_peaks():
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        d = json.loads(p.read_text())
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash(name):
    """Hash of a kernel's source file (name, or name:variant) and the shared header."""
    name = name.split(":")[0]
    h = hashlib.sha256()
    for f in sorted((ROOT / "sparse_attention_17_b200" / "csrc").glob("*")):
        if f.name in (name, "dsa_common.cuh"):
            h.update(f.read_bytes())
    return h.hexdigest()[:16]


def load_traffic(kernel_file):
    """DRAM traffic per launch from the committed ncu summary, if the kernel source has not
    changed since it was taken."""
    p = ROOT / "profiles" / "traffic.json"
    if not p.exists():
        return None
    d = json.loads(p.read_text()).get(kernel_file)
    if not d or d.get("source_hash") != kernel_source_hash(kernel_file):
        return None
    return d.get("bytes_per_launch_full")


class ClockSampler:
    """Samples SM clocks and throttle reasons with nvidia-smi during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.out = ""
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self):
        rows = []
        for line in (self.out or "").strip().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) != 8:
                continue
            try:
                rows.append((float(parts[0]), float(parts[1]), parts[3:]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for _, _, r in rows:
            for n, v in zip(names, r[1:]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(x[0] for x in rows),
                "sm_max_mhz": max(x[1] for x in rows), "reasons": sorted(reasons),
                "samples": len(rows)}


# ----------------------------------------------------------------------------------
# CPU oracle (baseline leg and reference arm)
# ----------------------------------------------------------------------------------
def oracle_rows_throughput(d, k, seconds, rng_seed=0, max_rows=None):
    """Runs the oracle's indexer + top-k + attention on blocks of consecutive query rows,
    each block starting at a uniformly drawn position of the workload, until about
    `seconds` of wall time are spent.  Each oracle call covers a whole block, so its
    OpenMP loop spreads the rows over all host threads.  Returns (rows/s, rows, threads,
    seconds)."""
    import numpy as np
    from oracle import oracle as O
    T = d["q_idx"].shape[0]
    r = np.random.default_rng(rng_seed)
    q_idx, k_idx, w = (O._f32(d[n]) for n in ("q_idx", "k_idx", "w"))
    fp8 = "kv_scale" in d
    q = d["q"]
    kv = d["kv"].numpy() if fp8 else O._f32(d["kv"])
    threads = O.num_threads()
    block = 2 * threads
    done, t0 = 0, time.perf_counter()
    while True:
        b0 = int(r.integers(0, T - block + 1))
        sc = O.indexer_scores_prefill(q_idx, k_idx, w, b0, block, b0 + block)
        idx = O.topk(sc, O.causal_n_valid(b0, block), k)
        if fp8:
            O.sparse_mla_fp8_prefill(q[b0:b0 + block], kv, d["kv_scale"], idx, 192 ** -0.5)
        else:
            O.sparse_mla_prefill(q[b0:b0 + block], kv, idx, 192 ** -0.5)
        done += block
        el = time.perf_counter() - t0
        if el >= seconds or (max_rows and done >= max_rows):
            return done / el, done, threads, el


# ----------------------------------------------------------------------------------
# native arm
# ----------------------------------------------------------------------------------
def run_native(args, rank, world, local_rank):
    import numpy as np
    import torch
    import torch.distributed as dist

    import sparse_attention_17_b200 as dsa
    from sparse_attention_17_b200 import inputs as G

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    plan = shard_plan(rank, world, args.T, args.topk)
    T, k = plan["T"], plan["topk"]
    fp8 = args.kv_dtype == "fp8"
    host = make_inputs(T, k, seed=plan["seed"], kv_dtype=args.kv_dtype)
    names = ("q_idx", "k_idx", "w", "q", "kv")
    x = {n: host[n].to(dev) for n in names}
    ld = (T + 3) // 4 * 4
    ws_bytes = dsa.layer_stack_workspace_size(T, args.window_rows)
    rw = max(16, ws_bytes // (4 * ld))
    rw = min(T, rw // 16 * 16 if rw > 16 else rw)
    scores = torch.empty((rw, ld), dtype=torch.float32, device=dev)
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    out = torch.empty((T, 16, 512), dtype=torch.bfloat16, device=dev)
    windows = [(q0, min(rw, T - q0)) for q0 in range(0, T, rw)]
    stream = torch.cuda.current_stream()

    def index_on(xin):
        """Indexer + top-k per window of query rows into the index buffer."""
        for q0, rows in windows:
            dsa.indexer_scores(xin["q_idx"], xin["k_idx"], xin["w"], scores, q0, rows)
            dsa.topk_select(scores, k, idx[q0:q0 + rows], q_begin=q0, rows=rows)

    def mla_on(xin, o, q0=0, rows=T):
        """Sparse MLA of queries q0 .. q0+rows-1 (their selected keys are cache rows)."""
        sl = slice(q0, q0 + rows)
        if fp8:
            dsa.sparse_mla_fp8_fwd(xin["q"][sl], xin["kv"], host["kv_scale"], idx[sl], o[sl],
                                   G.SCALE_MLA)
        else:
            dsa.sparse_mla_fwd(xin["q"][sl], xin["kv"], idx[sl], o[sl], G.SCALE_MLA)

    def step_on(xin, o, ev=None):
        """One prefill pass through the public C ABI: indexer + top-k per window of query
        rows into the index buffer, then sparse MLA over all queries."""
        if ev is not None:
            ev[0].record(stream)
        index_on(xin)
        if ev is not None:
            ev[1].record(stream)
        mla_on(xin, o)
        if ev is not None:
            ev[2].record(stream)

    def step(ev=None):
        step_on(x, out, ev)

    def sync_all():
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        step()
    assert dsa.check_device_errors() == 0
    sync_all()

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    launches0 = [dsa.launch_count(i) for i in range(dsa.KERNEL_KINDS)]
    with ClockSampler(local_rank) as clk:
        sync_all()
        start.record(stream)
        for i in range(args.steps):
            step(evs[i])
        stop.record(stream)
        torch.cuda.synchronize()
    launches = sum(dsa.launch_count(i) - launches0[i] for i in range(dsa.KERNEL_KINDS))
    ms_total = start.elapsed_time(stop)
    idx_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    mla_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    errs = dsa.check_device_errors()
    ms_total = max_over_ranks(ms_total, dev)

    # per-kernel split of the index phase (separate, untimed-for-value pass)
    e_idx = [torch.cuda.Event(enable_timing=True) for _ in range(2 * len(windows) + 1)]
    torch.cuda.synchronize()
    e_idx[0].record(stream)
    for i, (q0, rows) in enumerate(windows):
        dsa.indexer_scores(x["q_idx"], x["k_idx"], x["w"], scores, q0, rows)
        e_idx[2 * i + 1].record(stream)
        dsa.topk_select(scores, k, idx[q0:q0 + rows], q_begin=q0, rows=rows)
        e_idx[2 * i + 2].record(stream)
    torch.cuda.synchronize()
    indexer_ms = sum(e_idx[2 * i].elapsed_time(e_idx[2 * i + 1]) for i in range(len(windows)))
    topk_ms = sum(e_idx[2 * i + 1].elapsed_time(e_idx[2 * i + 2]) for i in range(len(windows)))

    # End to end through the API with host buffers (pinned): every step copies its inputs
    # host -> device and its output device -> host inside the timed region.  Steps are
    # pipelined the way a serving loop would run them: inputs and outputs are
    # double-buffered, the copies run on their own streams, and step i's upload and step
    # i-1's download overlap the computation of the step in between.
    e2e = None
    if not args.no_e2e:
        # the device-resident run's output, to check the pipelined steps against
        ref_out = out.cpu()
        pinned = {n: host[n].pin_memory() for n in names}
        h2d = sum(t.numel() * t.element_size() for t in pinned.values())
        xs = [x, {n: torch.empty_like(x[n]) for n in names}]
        outs = [out, torch.empty_like(out)]
        out_host = [torch.empty(out.shape, dtype=out.dtype, pin_memory=True) for _ in range(2)]
        d2h = out_host[0].numel() * out_host[0].element_size()
        s_up, s_down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        # as many steps as the device-timed run: the first upload and the last download
        # (pipeline fill and drain) are part of the measurement, spread over the K steps
        n_e2e = max(2, args.steps)

        # Within a step the copies are staged as the computation needs them: the indexer
        # inputs and the latent cache go up first and the index phase starts on them while
        # the 1.2 GB query block follows; the attention then runs per index window, and
        # each window's output rows go back while the next window is computed.
        early = [nme for nme in names if nme != "q"]

        def e2e_run(n):
            ev_early = [torch.cuda.Event() for _ in range(n)]
            ev_q = [torch.cuda.Event() for _ in range(n)]
            ev_comp = [torch.cuda.Event() for _ in range(n)]
            ev_down = [torch.cuda.Event() for _ in range(n)]
            for i in range(n):
                b = i % 2
                with torch.cuda.stream(s_up):
                    if i >= 2:
                        s_up.wait_event(ev_comp[i - 2])  # slot b's inputs are free again
                    for nme in early:
                        xs[b][nme].copy_(pinned[nme], non_blocking=True)
                    ev_early[i].record(s_up)
                    xs[b]["q"].copy_(pinned["q"], non_blocking=True)
                    ev_q[i].record(s_up)
                stream.wait_event(ev_early[i])
                if i >= 2:
                    stream.wait_event(ev_down[i - 2])  # slot b's output has been read
                index_on(xs[b])
                stream.wait_event(ev_q[i])
                ev_win = []
                for q0, rows in windows:
                    mla_on(xs[b], outs[b], q0, rows)
                    ev_win.append(torch.cuda.Event())
                    ev_win[-1].record(stream)
                ev_comp[i].record(stream)
                with torch.cuda.stream(s_down):
                    for (q0, rows), e in zip(windows, ev_win):
                        s_down.wait_event(e)
                        out_host[b][q0:q0 + rows].copy_(outs[b][q0:q0 + rows], non_blocking=True)
                    ev_down[i].record(s_down)
            stream.wait_event(ev_down[n - 1])

        e2e_run(2)
        sync_all()
        s2, t2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s2.record(stream)
        s_up.wait_event(s2)
        e2e_run(n_e2e)
        t2.record(stream)
        torch.cuda.synchronize()
        e2e_ms = s2.elapsed_time(t2) / n_e2e
        # the last two steps' outputs, read back through the pipeline, are the device run's
        outputs_match = all(torch.equal(out_host[b].view(torch.int16), ref_out.view(torch.int16))
                            for b in range(2))
        del ref_out
        e2e_ms = max_over_ranks(e2e_ms, dev)

        # the copies alone, each direction on its own stream: the host link's bound on e2e
        def copy_ms(fn, st, reps=3):
            fn()
            torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(st)
            for _ in range(reps):
                fn()
            b.record(st)
            torch.cuda.synchronize()
            return a.elapsed_time(b) / reps

        def up():
            with torch.cuda.stream(s_up):
                for nme in names:
                    xs[1][nme].copy_(pinned[nme], non_blocking=True)

        def down():
            with torch.cuda.stream(s_down):
                out_host[1].copy_(outs[1], non_blocking=True)

        h2d_ms = copy_ms(up, s_up)
        d2h_ms = copy_ms(down, s_down)

        def both():  # one step's upload and download at the same time, as in the pipeline
            up()
            down()

        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        stream.synchronize()
        a.record(stream)
        s_up.wait_event(a)
        s_down.wait_event(a)
        for _ in range(3):
            both()
        ev_u, ev_d = torch.cuda.Event(), torch.cuda.Event()
        ev_u.record(s_up)
        ev_d.record(s_down)
        stream.wait_event(ev_u)
        stream.wait_event(ev_d)
        b.record(stream)
        torch.cuda.synchronize()
        both_ms = a.elapsed_time(b) / 3
        e2e = {"value": aggregate_tokens_per_s(T, world, e2e_ms), "unit": UNIT,
               "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
               "steps": n_e2e,
               "overlap": "double-buffered inputs/outputs on their own copy streams; indexer "
                          "inputs first, queries second; attention and read-back per index window",
               "h2d_gbs_alone": round(h2d / (h2d_ms / 1e3) / 1e9, 1),
               "d2h_gbs_alone": round(d2h / (d2h_ms / 1e3) / 1e9, 1),
               "copy_bound_ms": round(max(h2d_ms, d2h_ms), 3),
               "copy_both_directions_ms": round(both_ms, 3),
               "outputs_match_device_run": outputs_match}

    result = None
    if rank == 0:
        work = algorithmic_work(T, k, kv_bytes=1 if fp8 else 2)
        peaks, peak_src = load_peaks()
        ms_step = ms_total / args.steps
        value = aggregate_tokens_per_s(T, world, ms_step)
        kern = {"indexer_ms": indexer_ms, "topk_ms": topk_ms, "sparse_mla_ms": mla_ms,
                "index_phase_ms": idx_ms}
        # dominant kernel
        if mla_ms >= indexer_ms:
            dom, flop, fname = "sparse_mla_mma_kernel", work["mla_flop"], "mla_mma.cu"
            dom_ms = mla_ms
        else:
            dom, flop, fname = "indexer_tc_kernel", work["indexer_flop"], "indexer_tc.cu"
            dom_ms = indexer_ms
        clocks = clk.summary()
        peak, peak_kind = choose_tensor_peak(peaks, clocks)
        achieved = flop / (dom_ms / 1e3) / 1e12
        gather_tbs = work["mla_gather_bytes"] / (mla_ms / 1e3) / 1e12
        step_roof_ms = (work["indexer_flop"] + work["mla_flop"]) / 1e12 / peak * 1e3
        roofline = {"kernel": dom, "bound": "tensor", "achieved": round(achieved, 2),
                    "peak": peak, "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                    "traffic": load_traffic(fname + (":fp8" if fp8 else "")),
                    "peak_source": f"{peak_src} bf16 dense, {peak_kind}",
                    "step_frac": round(step_roof_ms / ms_step, 4),
                    "step_roofline_ms": round(step_roof_ms, 3),
                    "l2_gather": {"achieved_tbs": round(gather_tbs, 3),
                                  "peak_tbs": L2_GATHER_PEAK_TBS,
                                  "frac": round(gather_tbs / L2_GATHER_PEAK_TBS, 4),
                                  "peak_source": L2_GATHER_PEAK_SOURCE}}
        others = {
            "indexer_tflops": round(work["indexer_flop"] / (indexer_ms / 1e3) / 1e12, 2),
            "indexer_frac_of_burst_peak": round(work["indexer_flop"] / (indexer_ms / 1e3) / 1e12
                                                / peaks.get("bf16_tflops", 1590.0), 4),
            "sparse_mla_tflops": round(work["mla_flop"] / (mla_ms / 1e3) / 1e12, 2),
            "sparse_mla_gather_gbs": round(work["mla_gather_bytes"] / (mla_ms / 1e3) / 1e9, 1),
            "topk_score_read_gbs": round(work["topk_read_bytes"] / (topk_ms / 1e3) / 1e9, 1),
        }
        result = {
            "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "fp8-e4m3 latent cache, f16 MMAs" if fp8 else "bf16",
            "data": "synthetic",
            "config": {"workload": f"dsa_prefill_T{T}_top{k}" + ("_fp8kv" if fp8 else ""),
                       "T": T, "topk": k, "kv_cache": "e4m3 x kv_scale" if fp8 else "bf16",
                       "batch_per_gpu": 1, "indexer_heads": 16, "indexer_dim": 64,
                       "heads": 16, "latent_dim": 576, "value_dim": 512,
                       "index_window_rows": rw, "parallelism": f"independent sequences x{world}",
                       "l2": "inputs larger than L2 (%.2f GB per step), no flush" %
                             (sum(t.numel() * t.element_size() for t in host.values()
                                  if hasattr(t, "numel")) / 1e9)},
            "roofline": roofline,
            "kernels": {kk: round(v, 4) for kk, v in kern.items()},
            "derived": others,
            "gpu_launches": launches,
            "clocks": clocks,
            "device_error_bits": errs,
        }
        if e2e is not None:
            e2e["value"] = round(e2e["value"], 1)
            e2e["ms_per_step"] = round(e2e["ms_per_step"], 3)
            result["e2e"] = e2e
        if not args.no_cpu_baseline and world == 1:
            rps, n, cores, el = oracle_rows_throughput(host, k, args.cpu_seconds)
            result["cpu_baseline"] = {
                "value": round(rps, 3), "unit": UNIT, "cores": cores, "kind": "oracle",
                "sample": f"{n} query rows of the T={T} workload in blocks of "
                          f"{2 * cores} consecutive rows at uniform positions (indexer + "
                          f"top-k + attention, fp64), {el:.1f} s"}
    return result


def run_rows(args, rank, world, local_rank):
    """One T-token prefill with its query rows split over the ranks (zig-zag blocks):
    each step all-gathers every rank's token shard of indexer keys and latent rows, then
    runs indexer + top-k + sparse MLA for the rank's own query blocks."""
    import torch
    import sparse_attention_17_b200 as dsa
    from sparse_attention_17_b200 import inputs as G
    from sparse_attention_17_b200 import sharding as SH
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    T, k = args.T, args.topk
    host = make_inputs(T, k, seed=0)  # one sequence: the same inputs on every rank
    x = {n: host[n].to(dev) for n in ("q_idx", "w", "q")}
    s0, ns = SH.token_shard(T, world, rank)
    k_local = host["k_idx"][s0:s0 + ns].to(dev)
    kv_local = host["kv"][s0:s0 + ns].to(dev)
    k_full = torch.empty((T, 64), dtype=torch.bfloat16, device=dev)
    kv_full = torch.empty((T, 576), dtype=torch.bfloat16, device=dev)
    blocks = SH.zigzag_blocks(T, world, rank)
    ld = (T + 3) // 4 * 4
    rw = max(16, dsa.layer_stack_workspace_size(T, args.window_rows) // (4 * ld)) // 16 * 16
    scores = torch.empty((rw, ld), dtype=torch.float32, device=dev)
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    out = torch.empty((T, 16, 512), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        SH.all_gather_rows(k_local, k_full)
        SH.all_gather_rows(kv_local, kv_full)
        SH.prefill_rank_rows(dsa, x["q_idx"], k_full, x["w"], x["q"], kv_full, blocks, k,
                             scores, idx, out, G.SCALE_MLA)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clk:
        a.record(stream)
        for _ in range(args.steps):
            step()
        b.record(stream)
        torch.cuda.synchronize()
    ms = max_over_ranks(a.elapsed_time(b) / args.steps, dev)
    errs = dsa.check_device_errors()
    if rank != 0:
        return None
    scored, attended = SH.pair_counts(blocks, k)
    return {"metric": METRIC, "value": round(T / (ms / 1e3), 1), "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "strong",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": f"dsa_prefill_T{T}_top{k}", "T": T, "topk": k,
                       "parallelism": f"query rows x{world} (zig-zag blocks, all-gather of "
                                      "k_idx and latent rows per step)",
                       "rank0_blocks": blocks, "rank0_scored_pairs": scored,
                       "rank0_attended_keys": attended},
            "clocks": clk.summary(), "device_error_bits": errs}


def _timed(step, steps, warmup, stream):
    """Device time of `steps` calls of step() after `warmup` calls (CUDA events)."""
    import torch
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        step()
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / steps


def run_decode(args, local_rank):
    """Batched sparse-MLA decode step: 64 sequences of 32768 cached tokens in 64-token
    pages; decode indexer over all cached keys + top-2048 + sparse MLA (split-k)."""
    import torch
    import sparse_attention_17_b200 as dsa
    from sparse_attention_17_b200 import inputs as G
    torch.cuda.set_device(local_rank)
    B, L, k = 64, 32768, args.topk
    fp8 = args.kv_dtype == "fp8"
    host = G.mla_decode_fp8(B=B, L=L, k=k) if fp8 else G.mla_decode(B=B, L=L, k=k)
    x = {n: host[n].cuda() for n in ("q_idx", "w", "k_idx_pool", "q", "kv_pool", "page_table",
                                      "seq_lens")}
    scores = torch.empty((B, L), dtype=torch.float32, device="cuda")
    idx = torch.empty((B, k), dtype=torch.int32, device="cuda")
    out = torch.empty((B, 16, 512), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(dsa.sparse_mla_workspace_size(B, k, decode=True) // 4 + 4, device="cuda")
    stream = torch.cuda.current_stream()

    def indexer():
        dsa.indexer_scores(x["q_idx"], x["k_idx_pool"], x["w"], scores,
                           page_table=x["page_table"], seq_lens=x["seq_lens"])

    def topk():
        dsa.topk_select(scores, k, idx, row_len=x["seq_lens"], max_len=L)

    def mla():
        if fp8:
            dsa.sparse_mla_fp8_fwd(x["q"], x["kv_pool"], host["kv_scale"], idx, out, G.SCALE_MLA,
                                   page_table=x["page_table"], seq_lens=x["seq_lens"],
                                   workspace=ws)
        else:
            dsa.sparse_mla_fwd(x["q"], x["kv_pool"], idx, out, G.SCALE_MLA,
                               page_table=x["page_table"], seq_lens=x["seq_lens"], workspace=ws)

    def step():
        indexer(); topk(); mla()

    ms = _timed(step, args.steps, args.warmup, stream)
    t_idx = _timed(indexer, args.steps, 1, stream)
    t_topk = _timed(topk, args.steps, 1, stream)
    t_mla = _timed(mla, args.steps, 1, stream)
    # the same step captured once as a CUDA graph (serving stacks replay decode steps so)
    side = torch.cuda.Stream()
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        step()
    stream.wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    ms_graph = _timed(graph.replay, args.steps, args.warmup, stream)
    assert dsa.check_device_errors() == 0
    peaks, src = load_peaks()
    gather = B * k * (576 if fp8 else 1152)
    kidx = B * L * 64 * 2
    # algorithmic HBM bytes of a step: indexer keys, the dense score row written and read
    # once, the gathered latent rows, queries, indices and outputs
    step_bytes = (kidx + 2 * B * L * 4 + gather + B * 16 * 576 * 2 + B * (16 * 64 * 2 + 16 * 4)
                  + B * k * 4 * 2 + B * 16 * 512 * 2)
    step_roof_ms = step_bytes / (peaks["hbm_gbs"] * 1e9) * 1e3
    return {"metric": "DSA decode sequences/sec (64 x 32768 paged, top-2048)", "value":
            round(B / (ms / 1e3), 1), "unit": "sequences/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True,
            "dtype": "fp8-e4m3 latent cache, f16 MMAs" if fp8 else "bf16", "data": "synthetic",
            "config": {"workload": "dsa_decode_B64_L32768_top2048" + ("_fp8kv" if fp8 else ""),
                       "page_size": 64, "kv_cache": "e4m3 x kv_scale" if fp8 else "bf16"},
            "kernels": {"indexer_ms": round(t_idx, 4), "topk_ms": round(t_topk, 4),
                        "sparse_mla_decode_ms": round(t_mla, 4)},
            "cuda_graph": {"ms_per_step": round(ms_graph, 4),
                           "value": round(B / (ms_graph / 1e3), 1)},
            "derived": {"indexer_key_read_gbs": round(kidx / (t_idx / 1e3) / 1e9, 1),
                        "mla_gather_gbs": round(gather / (t_mla / 1e3) / 1e9, 1),
                        "mla_gather_frac_of_hbm": round(gather / (t_mla / 1e3) / 1e9
                                                        / peaks["hbm_gbs"], 4),
                        "indexer_key_read_frac_of_hbm": round(kidx / (t_idx / 1e3) / 1e9
                                                              / peaks["hbm_gbs"], 4),
                        "step_hbm_bytes": step_bytes,
                        "step_hbm_roofline_ms": round(step_roof_ms, 4),
                        "step_frac_of_hbm_roofline": round(step_roof_ms / ms, 4),
                        "hbm_peak_gbs": peaks["hbm_gbs"], "peak_source": src}}


def run_varlen(args, local_rank):
    """Batched prefill of 16 independent prompts with lengths drawn uniformly from
    512..8192 tokens, packed along the token axis: dsa_index_varlen (indexer + top-k per
    sequence) and one sparse MLA over the packed batch."""
    import numpy as np
    import torch
    import sparse_attention_17_b200 as dsa
    from sparse_attention_17_b200 import inputs as G
    torch.cuda.set_device(local_rank)
    k = args.topk
    lens = [int(v) for v in np.random.default_rng(0).integers(512, 8193, 16)]
    starts = [int(v) for v in np.cumsum([0] + lens[:-1])]
    N = sum(lens)
    host = G.mla_prefill_gauss(T=N, seed=0, k=k)
    x = {n: host[n].cuda() for n in ("q_idx", "k_idx", "w", "q", "kv")}
    idx = torch.empty((N, k), dtype=torch.int32, device="cuda")
    out = torch.empty((N, 16, 512), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(dsa.index_varlen_workspace_size(max(lens), args.window_rows) // 4,
                     device="cuda")
    stream = torch.cuda.current_stream()

    def index():
        dsa.index_varlen(x["q_idx"], x["k_idx"], x["w"], starts, lens, k, idx, ws)

    def mla():
        dsa.sparse_mla_fwd(x["q"], x["kv"], idx, out, G.SCALE_MLA)

    def step():
        index(); mla()

    ms = _timed(step, args.steps, args.warmup, stream)
    t_idx = _timed(index, args.steps, 1, stream)
    t_mla = _timed(mla, args.steps, 1, stream)
    assert dsa.check_device_errors() == 0
    return {"metric": "DSA batched prefill tokens/sec (16 packed prompts, 512..8192 tokens, "
                      "top-2048)", "value": round(N / (ms / 1e3), 1), "unit": "tokens/s",
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms, 4), "higher_is_better": True, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": "dsa_varlen_prefill_16seq_top2048", "tokens": N,
                       "seq_lens": lens},
            "kernels": {"index_varlen_ms": round(t_idx, 4), "sparse_mla_ms": round(t_mla, 4)}}


def run_stack(args, local_rank):
    """The IndexCache stack: 27 layers "FSS" x 9 at T=16384, top-2048, through
    dsa_layer_stack (9 indexer + top-k passes, 27 sparse MLA passes)."""
    import torch
    import sparse_attention_17_b200 as dsa
    from sparse_attention_17_b200 import inputs as G
    torch.cuda.set_device(local_rank)
    T, k, pattern = 16384, args.topk, "FSS" * 9
    st = G.layer_stack(T=T, pattern=pattern, k=k)
    layers = [{n: v.cuda() for n, v in L.items()} for L in st["layers"]]
    outs = [torch.empty((T, 16, 512), dtype=torch.bfloat16, device="cuda") for _ in layers]
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    ws = torch.empty(dsa.layer_stack_workspace_size(T, args.window_rows) // 4, device="cuda")
    stream = torch.cuda.current_stream()
    dsa.reset_launch_counts()
    ms = _timed(lambda: dsa.layer_stack(pattern, layers, idx, ws, k, G.SCALE_MLA, outs),
                args.steps, args.warmup, stream)
    n_calls = args.steps + args.warmup
    launches = {kk: dsa.launch_count(i) // n_calls for i, kk in
                enumerate(["indexer", "topk", "attention", "combine"])}
    assert dsa.check_device_errors() == 0
    work = algorithmic_work(T, k)
    return {"metric": "IndexCache layer-stack tokens/sec (27 layers FSS x 9, T=16384, top-2048)",
            "value": round(T / (ms / 1e3), 1), "unit": "tokens/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3),
            "higher_is_better": True, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "dsa_indexcache_stack_T16384_FSSx9"},
            "launches_per_call": launches,
            "derived": {"tflop_per_call": round((9 * work["indexer_flop"] + 27 * work["mla_flop"])
                                                / 1e12, 2)}}


def run_reference(args, rank, world):
    """The CPU oracle, as it stands, on bounded samples of the same workload."""
    if rank != 0:
        return None
    T, k = args.T, args.topk
    host = make_inputs(T, k, seed=0)
    per_step = max(1.0, min(args.cpu_seconds, 120.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_rows_throughput(host, k, per_step / 4, rng_seed=1)
    vals, rows, secs = [], 0, 0.0
    cores = 1
    for i in range(args.steps):
        rps, n, cores, el = oracle_rows_throughput(host, k, per_step, rng_seed=100 + i)
        vals.append(rps)
        rows += n
        secs += el
    value = rows / secs
    return {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": 0,
        # a step is the whole T-token prefill, at the sampled rate: extrapolated from the
        # sampled rows, not timed as a whole
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(T * 1e3 / value, 3),
        "extrapolated": True,
        "sampled_ms_per_step": round(secs * 1e3 / max(1, args.steps), 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "impl": "reference",
        "config": {"workload": f"dsa_prefill_T{T}_top{k}", "T": T, "topk": k},
        "cpu_baseline": {"value": round(value, 3), "unit": UNIT, "cores": cores,
                         "kind": "oracle",
                         "sample": f"{rows} query rows of the T={T} workload in blocks of "
                                   f"{2 * cores} consecutive rows at uniform positions, "
                                   f"{secs:.1f} s over {args.steps} steps"},
        "e2e": {"value": round(value, 3), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    args = parse_args(argv)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return 0
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600))
    try:
        if args.workload == "decode":
            res = run_decode(args, local_rank) if rank == 0 else None
        elif args.workload == "stack":
            res = run_stack(args, local_rank) if rank == 0 else None
        elif args.workload == "varlen":
            res = run_varlen(args, local_rank) if rank == 0 else None
        elif args.shard == "rows":
            res = run_rows(args, rank, world, local_rank)
        else:
            res = run_native(args, rank, world, local_rank)
            if world > 1 and not args.no_rows:
                # the same prefill split over the ranks by query rows (every rank takes part)
                rows_line = run_rows(args, rank, world, local_rank)
                if res is not None:
                    res["strong_scaling"] = {kk: rows_line[kk] for kk in
                                             ("value", "unit", "ms_per_step", "scaling", "config")}
            if world == 1 and res is not None and not args.no_decode:
                # the batched decode workload, measured in the same run (a nested object,
                # so that the line stays one line)
                import torch
                torch.cuda.synchronize()
                dec = run_decode(args, local_rank)
                res["decode"] = {kk: dec[kk] for kk in ("metric", "value", "unit", "ms_per_step",
                                                       "kernels", "cuda_graph", "derived",
                                                       "config")}
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    if res is not None:
        print(json.dumps(res), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
