"""Benchmark: one step = plan -> dispatch -> combine over one batch of seeded
synthetic routing, through the libmoonep C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl moonep|reference]
                    [--workload hot] [--alpha A] [--rule 0|1|2] [--no-sweep] [--sweep FILE]

Prints one JSON line (rank 0).  Timing: W untimed warm-up steps; then K steps,
each preceded by an L2 flush (a 512 MiB memset, then a 256 MiB read so that the
memset's dirty lines leave L2 before the step; both outside the step's events) and
bracketed by CUDA events on the launching stream; a barrier and a device
synchronise on both sides of the timed loop; the max over ranks.  value =
routed (token, k) rows of all ranks / step time.  N > 1 runs N independent
replicas (each rank its own layer, seed + rank): the path has no exchange step
on one GPU, so no collective is on the data path.
"""
import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = ("dispatch+combine GB/s (% of HBM peak) and routed tokens/s vs maxvio; plan µs")
UNIT = "routed tokens/s"
FLUSH_BYTES = 512 << 20   # written between steps: larger than the 126 MB L2
FLUSH_READ_BYTES = 256 << 20  # then read, so the flush's dirty lines are written back
                              # before the step starts and are not charged to it
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "traffic.json")


# ---------------------------------------------------------------- helpers
def algorithmic_bytes(cfgd):
    """Bytes each kernel must move (read each input once, write each output
    once, index traffic included)."""
    R, S, K, H = cfgd["R"], cfgd["S"], cfgd["K"], cfgd["H"]
    T, P = R * S, R * S * K
    fp8 = cfgd.get("payload") == "fp8"
    row_out = H + (H // 128) * 4 if fp8 else 2 * H
    return dict(
        plan=12 * P,
        dispatch=T * H * 2 + P * row_out + 4 * P,
        combine=P * H * 2 + T * H * 2 + 8 * P,
    )


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def kernel_source_hash(name):
    src = os.path.join(ROOT, "dispatch_moonep_plan_b200", "csrc", name)
    return hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]


def profiled_traffic(kernel, workload):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the kernel source as it is now; else None."""
    if not os.path.exists(PROFILE_TRAFFIC):
        return None
    d = json.load(open(PROFILE_TRAFFIC)).get("%s/%s" % (kernel, workload))
    if not d or d.get("source_sha") != kernel_source_hash(d["source"]):
        return None
    return d["dram_bytes_per_launch"]


class ClockSampler:
    """Samples SM clock and clock-event reasons with NVML while running."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, index, period=0.005):
        self.index, self.period = index, period
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._t = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit and bit != 0x1:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nv is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._t:
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def dist_setup(args):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def reduce_max(values, world):
    """Max over ranks of a list of floats (host plumbing for the timing)."""
    if world == 1:
        return list(values)
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor(values, dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.cpu().tolist()


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def rank_seed(base, rank):
    return base + 1000 * rank


# ---------------------------------------------------------------- oracle arm
def oracle_sample_step(cfgd, idx, w, x_rows, rule, tokens):
    """One step of the oracle on a bounded sample of the workload: the full
    plan over all P picks, then dispatch, the identity stand-in expert and
    combine of the sampled tokens only.  x_rows [n, H] holds the sampled
    tokens' hidden states (bf16 bits).  Returns the seconds of each part."""
    import numpy as np

    import oracle
    R, S, E, K, B = (cfgd[k] for k in ("R", "S", "E", "K", "B"))
    C = S * K
    fp8 = cfgd.get("payload") == "fp8"
    tokens = np.asarray(tokens, np.int64)
    t0 = time.perf_counter()
    pl = oracle.plan(R, S, E, K, B, idx, rule=rule)
    t1 = time.perf_counter()
    if pl["status"] != 0:
        raise SystemExit("oracle plan failed with status %d (rule %d)" % (pl["status"], rule))
    # a source map into the compact x_rows (harness bookkeeping, not timed)
    rows = pl["dst_row"][tokens].reshape(-1).astype(np.int64)
    src_c = np.zeros(R * S * K, np.int32)
    src_c[rows] = np.arange(rows.size, dtype=np.int32)
    t2 = time.perf_counter()
    if fp8:
        q, sc = oracle.dispatch_rows_fp8(K, x_rows, src_c, rows)
    else:
        recv = oracle.dispatch_rows(K, x_rows, src_c, rows)
    t3 = time.perf_counter()
    if fp8:
        eo = oracle.expert_rows("identity", E, B, C, pl, rows, q=q, s=sc)
    else:
        eo = oracle.expert_rows("identity", E, B, C, pl, rows, recv_bits=recv)
    t4 = time.perf_counter()
    oracle.combine_tokens(np.asarray(w, np.float32)[tokens], eo.reshape(tokens.size, K, -1))
    t5 = time.perf_counter()
    return dict(plan=t1 - t0, dispatch=t3 - t2, expert=t4 - t3, combine=t5 - t4,
                tokens=int(tokens.size))


def oracle_rates(cfgd, parts):
    """Measured seconds of a sample step, and the whole-workload step the
    sample stands for (the plan already covers every pick; the per-token
    parts scale with T / sampled tokens)."""
    T = cfgd["R"] * cfgd["S"]
    per_tok = parts["dispatch"] + parts["expert"] + parts["combine"]
    measured = parts["plan"] + per_tok
    full = parts["plan"] + per_tok * T / parts["tokens"]
    return measured, full


def calibrate_tokens(cfgd, idx, w, x_pool_fn, rule, budget_s, rng):
    """Sampled-token count whose oracle step takes about budget_s seconds."""
    T = cfgd["R"] * cfgd["S"]
    n0 = min(256, T)
    toks = rng.choice(T, size=n0, replace=False)
    p = oracle_sample_step(cfgd, idx, w, x_pool_fn(n0), rule, toks)
    per_tok = (p["dispatch"] + p["expert"] + p["combine"]) / n0
    n = int((budget_s - p["plan"]) / max(per_tok, 1e-9))
    return max(n0, min(T, n))


def host_cpu():
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return dict(cpu_model=model, nproc=os.cpu_count())


def run_reference(args, cfgd):
    """The CPU oracle as the reference arm (rank 0 only).  Each step is the
    oracle on a bounded sample of the workload (full plan, sampled tokens'
    dispatch/expert/combine), sized to about 1.5 s; ms_per_step is the
    measured time of those steps."""
    import numpy as np

    from dispatch_moonep_plan_b200 import workloads as wl
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    oracle.lib()
    T, P, H = cfgd["R"] * cfgd["S"], cfgd["R"] * cfgd["S"] * cfgd["K"], cfgd["H"]
    idx, w = wl.routing(cfgd, seed=rank_seed(0, 0), alpha=args.alpha)
    rng = np.random.default_rng(0)
    pool = {}

    def x_pool(n):
        # hidden states for the sampled tokens (same N(0,1) bf16 law as the
        # GPU arm's x; drawn for the sample only)
        if pool.get("n", 0) < n:
            pool["x"] = wl.bf16_bits(wl.hidden(n, H, seed=0))
            pool["n"] = n
        return pool["x"][:n]

    n_tok = calibrate_tokens(cfgd, idx, w, x_pool, args.rule, 1.5, rng)
    xs = x_pool(n_tok)
    for _ in range(args.warmup):
        oracle_sample_step(cfgd, idx, w, xs, args.rule, rng.choice(T, n_tok, replace=False))
    measured, full, parts = [], [], None
    t0 = time.perf_counter()
    for _ in range(args.steps):
        parts = oracle_sample_step(cfgd, idx, w, xs, args.rule,
                                   rng.choice(T, n_tok, replace=False))
        m, f = oracle_rates(cfgd, parts)
        measured.append(m)
        full.append(f)
    wall = time.perf_counter() - t0
    step_s = statistics.mean(measured)
    full_s = statistics.mean(full)
    value = P / full_s
    sample = ("each step: the full oracle plan over all %d picks, then dispatch + identity "
              "expert + combine of %d of the %d tokens (a fresh random sample each step); "
              "ms_per_step is the measured time of such a step; value = all %d picks / the "
              "whole-workload step time that the sample stands for (plan time + per-token time "
              "x %d tokens), given under 'extrapolated'" % (P, n_tok, T, P, T))
    line = dict(impl="reference", metric=METRIC, value=value, unit=UNIT, n_gpus=args.gpus,
                steps=args.steps, warmup=args.warmup, ms_per_step=step_s * 1e3,
                higher_is_better=True, scaling="weak", vs_baseline=None, dtype="bf16",
                data="synthetic", config=workload_config(cfgd, args),
                cpu_baseline=dict(kind="oracle", value=value, unit=UNIT, cores=1, sample=sample,
                                  sampled_tokens=n_tok,
                                  last_step_s={k: v for k, v in parts.items() if k != "tokens"},
                                  **host_cpu()),
                extrapolated=dict(ms_per_full_step=full_s * 1e3, picks_per_full_step=P,
                                  how="plan seconds + sampled per-token seconds x T / n"),
                e2e=dict(value=value, unit=UNIT, h2d_bytes_per_step=0, d2h_bytes_per_step=0),
                wall_s=wall)
    print(json.dumps(line), flush=True)


def workload_config(cfgd, args):
    c = dict(workload=cfgd["name"], R=cfgd["R"], S=cfgd["S"], E=cfgd["E"], K=cfgd["K"],
             B=cfgd["B"], H=cfgd["H"], payload=cfgd.get("payload", "bf16"),
             routing=cfgd["routing"], rule=args.rule,
             l2="flushed before every step (512 MiB memset + 256 MiB read, outside the "
                "step's events)")
    if cfgd["routing"] == "zipf":
        c["alpha"] = args.alpha if args.alpha is not None else cfgd["alpha"]
    if cfgd["routing"] == "logits":
        c["sigma"] = cfgd["sigma"]
    return c


# ---------------------------------------------------------------- GPU arm
def run_gpu(args, cfgd, emit=True):
    import numpy as np
    import torch

    from dispatch_moonep_plan_b200 import moonep as me
    from dispatch_moonep_plan_b200 import workloads as wl

    world, rank, local = dist_setup(args) if emit else (1, 0, torch.cuda.current_device())
    seed = rank_seed(0, rank)
    cfg = me.config_from(cfgd, args.rule)
    s = me.sizes(cfg)
    T, P, H, K = s.tokens, s.picks, cfg.H, cfg.K
    fp8 = cfg.payload == me.PAYLOAD_FP8
    idx_np, w_np = wl.routing(cfgd, seed=seed, alpha=args.alpha)
    x = wl.hidden(T, H, seed=seed, device="cuda")
    idx = torch.from_numpy(idx_np).cuda()
    w = torch.from_numpy(w_np).cuda()
    bufs = me.PlanBuffers(cfg)
    if fp8:
        recv = torch.empty((P, H), dtype=torch.uint8, device="cuda")
        scale = torch.empty((P, H // 128), dtype=torch.float32, device="cuda")
        eo = torch.empty((P, H), dtype=torch.bfloat16, device="cuda")
    else:
        recv = torch.empty((P, H), dtype=torch.bfloat16, device="cuda")
        scale = None
        eo = recv  # identity expert: combine reads the receive buffers in place
    y = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    flush_w = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    flush_r = torch.zeros(FLUSH_READ_BYTES // 4, dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()

    warm = getattr(args, "warm_l2", False)

    def flush():
        if warm:  # sweep-only: the tiny workload fits in L2 and is also timed warm
            return
        flush_w.zero_()
        flush_r.sum()

    def step(ev=None, st=None):
        st = stream if st is None else st
        if ev:
            ev[0].record(st)
        me.plan(cfg, idx, bufs, st)
        if ev:
            ev[1].record(st)
        me.dispatch(cfg, bufs, x, recv, scale, st)
        if ev:
            ev[2].record(st)
        if fp8:
            me.expert_standin(cfg, bufs, recv, scale, me.EXPERT_IDENTITY, eo, st)
        if ev:
            ev[3].record(st)
        me.combine(cfg, bufs, eo, w, y, st)
        if ev:
            ev[4].record(st)

    for _ in range(args.warmup):
        flush()
        step()
    torch.cuda.synchronize()
    st = me.plan_status(bufs, stream)
    if st[0] != me.STATUS_OK:
        raise SystemExit("plan failed with status %s (rule %d); try --rule 1" % (st, args.rule))
    maxvio = float(bufs.maxvio.item())

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    region = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    with ClockSampler(local) as clk:
        barrier(world)
        torch.cuda.synchronize()
        region[0].record(stream)
        for i in range(args.steps):
            flush()
            step(evs[i])
        region[1].record(stream)
        torch.cuda.synchronize()
        barrier(world)
    t_plan = [e[0].elapsed_time(e[1]) for e in evs]
    t_disp = [e[1].elapsed_time(e[2]) for e in evs]
    t_comb = [e[3].elapsed_time(e[4]) for e in evs]
    t_step = [a + b + c for a, b, c in zip(t_plan, t_disp, t_comb)]
    region_ms = region[0].elapsed_time(region[1])
    # per-kernel figures: the median of the K steps (a host stall between two
    # event records lands in one interval and would move a mean), then the
    # max over ranks; the means and the slowest step are kept beside them
    m_plan, m_disp, m_comb, m_step = (statistics.median(v) for v in (t_plan, t_disp, t_comb, t_step))
    mean = dict(plan_us=statistics.mean(t_plan) * 1e3, dispatch_us=statistics.mean(t_disp) * 1e3,
                combine_us=statistics.mean(t_comb) * 1e3, step_ms=statistics.mean(t_step),
                slowest_step_ms=max(t_step))
    m_plan, m_disp, m_comb, m_step, region_ms = reduce_max(
        [m_plan, m_disp, m_comb, m_step, region_ms], world)

    # ---- the same step as one CUDA graph, events only around each replay ----
    # (the per-kernel pass above puts events between the kernels; the headline
    # step time comes from this pass when the capture works)
    if fp8:
        # the fp8 step has the (untimed) stand-in dequantise between dispatch
        # and combine; a graph would time it too, so keep the per-kernel events
        clk_g, m_graph = clk, None
        graph_note = ("sum of the plan, dispatch and combine event intervals (the stand-in "
                      "expert between them is not part of the step)")
    else:
        with ClockSampler(local) as clk_g:
            m_graph, graph_note = graph_step_time(step, flush, args, world, stream)
    step_ms = m_graph if m_graph is not None else m_step
    clocks = clk_g.summary() if m_graph is not None else clk.summary()
    # each kernel's interval inside one captured step, events as graph nodes
    ig = graph_node_times(lambda ev, st: step(ev, st), 5, flush, args, stream)
    ig = reduce_max(ig if ig else [float("nan")] * 4, world)

    # ---- end to end through the C ABI with host buffers ----
    if getattr(args, "no_e2e", False):
        e2e = dict(ms=float("nan"), serial_ms=float("nan"), h2d=0, d2h=0)
    else:
        e2e = e2e_pipelined(me, cfg, bufs, x, idx, w, recv, scale, eo, fp8, args, world)

    bytes_ = algorithmic_bytes(cfgd)
    peak, peak_kind = peaks()
    disp_gbs = bytes_["dispatch"] / (m_disp * 1e-3) / 1e9
    comb_gbs = bytes_["combine"] / (m_comb * 1e-3) / 1e9
    dom = "dispatch" if m_disp >= m_comb else "combine"
    dom_gbs = disp_gbs if dom == "dispatch" else comb_gbs
    traffic = profiled_traffic(dom, cfgd["name"])
    value = world * P / (step_ms * 1e-3)
    out = dict(
        metric=METRIC, value=value, unit=UNIT, n_gpus=world, steps=args.steps,
        warmup=args.warmup, ms_per_step=step_ms, higher_is_better=True, scaling="weak",
        vs_baseline=None, dtype="fp8" if fp8 else "bf16",
        data="synthetic (seeded routing and N(0,1) hidden states; one independent layer per GPU)",
        config=workload_config(cfgd, args),
        roofline=dict(bound="hbm", kernel=dom, achieved=dom_gbs, peak=peak, unit="GB/s",
                      frac=dom_gbs / peak, traffic=traffic,
                      algorithmic_bytes=bytes_[dom], peak_kind=peak_kind),
        plan_us=m_plan * 1e3, dispatch_us=m_disp * 1e3, combine_us=m_comb * 1e3,
        in_graph=dict(plan_us=ig[0], dispatch_us=ig[1], combine_us=ig[3],
                      how="the step captured once as a CUDA graph with its events as graph "
                          "nodes between the kernels; median of the K replays (L2 flushed "
                          "before each); the keys above time each kernel by events on the "
                          "stream around its own launch"),
        dispatch_GBps=disp_gbs, combine_GBps=comb_gbs,
        dispatch_frac=disp_gbs / peak, combine_frac=comb_gbs / peak,
        maxvio=maxvio, tokens_per_s=world * T / (step_ms * 1e-3),
        step_timing=graph_note, step_ms_per_kernel_events=m_step,
        region_ms=region_ms, stat="median of the K timed steps, max over ranks", mean=mean,
        e2e=dict(value=world * P / (e2e["ms"] * 1e-3), unit=UNIT,
                 h2d_bytes_per_step=e2e["h2d"], d2h_bytes_per_step=e2e["d2h"],
                 ms_per_step=e2e["ms"], serial_ms_per_step=e2e["serial_ms"],
                 how="pinned host x/idx/w in and y out every step; the next step's "
                     "inputs copy in and the previous step's y copies out on two copy "
                     "streams while the step computes"),
        gpu_launches=(4 if fp8 else 3) * args.steps,
        clocks=clocks, clocks_per_kernel_pass=clk.summary(),
    )
    if emit and not args.no_side:
        out["backward"] = measure_backward(me, cfg, bufs, T, P, H, K, flush, world, eo)
        out["side"] = measure_side(me, wl, flush, world)
        out["expert_gemm"] = measure_gemm(me, wl, flush, world, local=local)
        out["expert_gemm_fp8"] = measure_gemm_fp8(me, wl, flush, world, local=local)
    if rank == 0 and emit and world == 1 and not args.no_cpu_baseline:
        cb = cpu_baseline(cfgd, idx_np, w_np, x, args.rule)
        out["cpu_baseline"] = cb
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return out if rank == 0 else None


def graph_node_times(body, n_events, flush, args, stream):
    """Capture body(events, stream) once as a CUDA graph whose events are
    graph nodes, replay it W + K times (L2 flushed before each, outside the
    graph) and return the median of each interval between consecutive events
    over the K timed replays, in µs; None if the capture is not supported."""
    import torch
    try:
        ev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(n_events)]
        cs = torch.cuda.Stream()
        cs.wait_stream(stream)
        with torch.cuda.stream(cs):
            body(ev, cs)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cs):
            body(ev, cs)
        torch.cuda.synchronize()
    except Exception:
        return None
    iv = [[] for _ in range(n_events - 1)]
    for i in range(args.warmup + args.steps):
        flush()
        g.replay()
        torch.cuda.synchronize()
        if i >= args.warmup:
            for j in range(n_events - 1):
                iv[j].append(ev[j].elapsed_time(ev[j + 1]) * 1e3)
    del g
    return [statistics.median(v) for v in iv]


def graph_step_time(step, flush, args, world, stream):
    """Capture plan -> dispatch -> combine once as a CUDA graph, then time K
    replays (L2 flushed before each, outside the events).  Returns (mean ms or
    None, a note saying how the step was timed)."""
    import torch
    try:
        cs = torch.cuda.Stream()
        cs.wait_stream(stream)
        with torch.cuda.stream(cs):
            step(st=cs)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cs):
            step(st=cs)
        torch.cuda.synchronize()
    except Exception as e:  # capture unsupported: keep the per-kernel-event step time
        return None, "sum of per-kernel event intervals (graph capture failed: %s)" % e
    for _ in range(args.warmup):
        flush()
        g.replay()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    cur = torch.cuda.current_stream()
    for a, b in evs:
        flush()
        a.record(cur)
        g.replay()
        b.record(cur)
    torch.cuda.synchronize()
    barrier(world)
    m = statistics.median(a.elapsed_time(b) for a, b in evs)
    m = reduce_max([m], world)[0]
    del g
    return m, ("one CUDA graph of plan -> dispatch -> combine per step, CUDA events around "
               "each replay, L2 flushed before each outside the events; the median of the K "
               "replays")


def e2e_pipelined(me, cfg, bufs, x, idx, w, recv, scale, eo, fp8, args, world):
    """The step through the C ABI from pinned host buffers: every step copies
    its own x, idx and w in and its y out.  Inputs and outputs are double
    buffered on the device; H2D of step i+1 and D2H of step i-1 run on two
    copy streams while step i computes.  Also times the plain serial loop."""
    import torch
    T, H, K = x.shape[0], x.shape[1], idx.shape[1]
    cs = torch.cuda.current_stream()
    h2d_s, d2h_s = torch.cuda.Stream(), torch.cuda.Stream()
    x_h = x.cpu().pin_memory()
    idx_h = idx.cpu().pin_memory()
    w_h = w.cpu().pin_memory()
    y_h = [torch.empty((T, H), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    xs = [x, torch.empty_like(x)]
    idxs = [idx, torch.empty_like(idx)]
    ws = [w, torch.empty_like(w)]
    ys = [torch.empty((T, H), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    h2d = x_h.numel() * 2 + idx_h.numel() * 4 + w_h.numel() * 4
    d2h = y_h[0].numel() * 2
    n = max(4, min(args.steps, 50))

    def compute(sl):
        me.plan(cfg, idxs[sl], bufs, cs)
        me.dispatch(cfg, bufs, xs[sl], recv, scale, cs)
        if fp8:
            me.expert_standin(cfg, bufs, recv, scale, me.EXPERT_IDENTITY, eo, cs)
        me.combine(cfg, bufs, eo, ws[sl], ys[sl], cs)

    def copy_in(sl):
        xs[sl].copy_(x_h, non_blocking=True)
        idxs[sl].copy_(idx_h, non_blocking=True)
        ws[sl].copy_(w_h, non_blocking=True)

    def run(steps, timed):
        ev = lambda: torch.cuda.Event(enable_timing=timed)  # noqa: E731
        in_ready = [ev(), ev()]
        in_free = [ev(), ev()]
        out_ready = [ev(), ev()]
        out_free = [ev(), ev()]
        for e_ in in_free + out_free:
            e_.record(cs)
        start, end = ev(), ev()
        start.record(cs)
        h2d_s.wait_event(start)
        with torch.cuda.stream(h2d_s):
            copy_in(0)
            in_ready[0].record(h2d_s)
        for i in range(steps):
            sl = i % 2
            if i + 1 < steps:
                nx = (i + 1) % 2
                h2d_s.wait_event(in_free[nx])
                with torch.cuda.stream(h2d_s):
                    copy_in(nx)
                    in_ready[nx].record(h2d_s)
            cs.wait_event(in_ready[sl])
            cs.wait_event(out_free[sl])
            compute(sl)
            in_free[sl].record(cs)
            out_ready[sl].record(cs)
            d2h_s.wait_event(out_ready[sl])
            with torch.cuda.stream(d2h_s):
                y_h[sl].copy_(ys[sl], non_blocking=True)
                out_free[sl].record(d2h_s)
        cs.wait_event(out_free[(steps - 1) % 2])
        cs.wait_event(out_free[(steps - 2) % 2])
        end.record(cs)
        torch.cuda.synchronize()
        return start.elapsed_time(end) / steps if timed else None

    run(3, False)
    barrier(world)
    ms = run(n, True)
    # the plain serial loop, for comparison
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(cs)
    for _ in range(n):
        copy_in(0)
        compute(0)
        y_h[0].copy_(ys[0], non_blocking=True)
    e1.record(cs)
    torch.cuda.synchronize()
    barrier(world)
    ms, serial = reduce_max([ms, e0.elapsed_time(e1) / n], world)
    return dict(ms=ms, serial_ms=serial, h2d=h2d, d2h=d2h)


def measure_backward(me, cfg, bufs, T, P, H, K, flush, world, eo, reps=10):
    """Backward of combine (d_expert_out = w * dy per row, d_w = <dy, row>) and
    of dispatch (dx = sum of the token's K rows) on the bench's workload.  eo
    is the step's bf16 expert output [P, H] (the forward's combine input)."""
    import torch

    from dispatch_moonep_plan_b200 import workloads as wl
    dy = wl.hidden(T, H, seed=77, device="cuda")
    w = torch.rand((T, K), device="cuda")
    d_eo = torch.empty_like(eo)
    d_w = torch.empty((T, K), dtype=torch.float32, device="cuda")
    dx = torch.empty_like(dy)
    peak, _ = peaks()

    def timeit(fn):
        ts = []
        for i in range(reps + 2):
            flush()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            if i >= 2:
                ts.append(a.elapsed_time(b))
        return reduce_max([statistics.median(ts)], world)[0]

    tc = timeit(lambda: me.combine_backward(cfg, bufs, dy, eo, w, d_eo, d_w))
    td = timeit(lambda: me.dispatch_backward(cfg, bufs, eo, dx))
    cb = T * H * 2 + 2 * P * H * 2 + P * 4 + 8 * P
    db = P * H * 2 + T * H * 2 + 4 * P
    out = dict(combine_backward_us=tc * 1e3, combine_backward_GBps=cb / tc / 1e6,
               combine_backward_frac=cb / tc / 1e6 / peak,
               dispatch_backward_us=td * 1e3, dispatch_backward_GBps=db / td / 1e6,
               dispatch_backward_frac=db / td / 1e6 / peak)
    del dy, d_eo, dx
    torch.cuda.empty_cache()
    return out


def measure_side(me, wl, flush, world, reps=10, S=None, Hp=None, rule=0):
    """Replica prefetch (bf16 weights) and replica grad-reduce (fp32 grads) at
    the fp8 workload's sizes on VMM-aliased [E+B, H, H'] views (S, if given,
    shrinks only the routing that places the slots; Hp the weight rows)."""
    import numpy as np
    import torch
    kw = {}
    if S:
        kw["S"] = S
    if Hp:
        kw["Hp"] = Hp
    cfgd = wl.cfg_with("fp8", **kw)
    cfg = me.config_from(cfgd, rule)
    idx, _ = wl.routing(cfgd, seed=0)
    bufs = me.PlanBuffers(cfg)
    me.plan(cfg, torch.from_numpy(idx).cuda(), bufs)
    torch.cuda.synchronize()
    st = me.plan_status(bufs)
    if st[0] != me.STATUS_OK:
        return dict(failed="plan status %s" % st)
    se = bufs.slot_expert.cpu().numpy()[:cfg.R * cfg.B]
    used = se[se >= 0]
    n_used = int(used.size)
    reps_per_e = np.bincount(used, minlength=cfg.E)
    E, B, H, Hp = cfg.E, cfg.B, cfg.H, cfg.Hp
    peak, _ = peaks()

    def timeit(fn):
        ts = []
        for i in range(reps + 2):
            flush()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            if i >= 2:
                ts.append(a.elapsed_time(b))
        return reduce_max([statistics.median(ts)], world)[0]

    out = dict(workload=cfgd["name"] + " H'=%d" % Hp, used_slots=n_used,
               replicated_experts=int((reps_per_e > 0).sum()))
    wv = me.WeightViews(cfg, elem_bytes=2)
    try:
        v0 = me.weight_view_tensor(wv, 0, cfg, torch.bfloat16)
        v0[:E].normal_()
        torch.cuda.synchronize()
        t = timeit(lambda: me.prefetch(cfg, bufs, wv.ptrs, 2))
        nbytes = n_used * 2 * H * Hp * 2
        out.update(prefetch_us=t * 1e3, prefetch_GBps=nbytes / t / 1e6,
                   prefetch_frac=nbytes / t / 1e6 / peak, prefetch_bytes=nbytes)
        del v0
    finally:
        wv.close()
    gv = me.WeightViews(cfg, elem_bytes=4)
    try:
        for r in range(cfg.R):
            me.weight_view_tensor(gv, r, cfg, torch.float32)[E if r else 0:].normal_()
        torch.cuda.synchronize()
        t = timeit(lambda: me.grad_reduce(cfg, bufs, gv.ptrs))
        nbytes = int(sum((2 + n) * H * Hp * 4 for n in reps_per_e if n > 0))
        out.update(grad_reduce_us=t * 1e3, grad_reduce_GBps=nbytes / t / 1e6,
                   grad_reduce_frac=nbytes / t / 1e6 / peak, grad_reduce_bytes=nbytes)
    finally:
        gv.close()
    torch.cuda.empty_cache()
    return out


def tensor_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return float(d["bf16_tflops"]), float(d["bf16_tflops_sustained"]), "measured"
    return 1590.0, 1400.0, "fallback"


def measure_gemm(me, wl, flush, world, reps=5, S=None, local=None, rule=0, base="fp8", Hp=None):
    """The grouped expert GEMM that consumes the plan, by default at the fp8
    workload's sizes with a bf16 payload (R16 S16384 E128 K8 H4096 B8,
    H'=1536): recv [R*C, H] bf16, VMM-aliased [E+B, H, H'] weight views
    filled by the replica prefetch, out [R*C, H'] bf16.  2*R*C*H*H' FLOPs per
    launch.  `base` and `Hp` pick another workload's routing and sizes."""
    import torch
    kw = {"payload": "bf16"}
    if S:
        kw["S"] = S
    if Hp or not wl.WORKLOADS[base]["Hp"]:
        kw["Hp"] = Hp or 1536
    cfgd = wl.cfg_with(base, **kw)
    cfg = me.config_from(cfgd, rule)
    idx, _ = wl.routing(cfgd, seed=0)
    bufs = me.PlanBuffers(cfg)
    me.plan(cfg, torch.from_numpy(idx).cuda(), bufs)
    torch.cuda.synchronize()
    st = me.plan_status(bufs)
    if st[0] != me.STATUS_OK:
        return dict(failed="plan status %s (rule %d)" % (st, rule))
    R, E, H, Hp = cfg.R, cfg.E, cfg.H, cfg.Hp
    P = R * cfg.S * cfg.K
    recv = wl.hidden(P, H, seed=1, device="cuda")
    y = torch.empty((P, Hp), dtype=torch.bfloat16, device="cuda")
    views = me.WeightViews(cfg, elem_bytes=2)
    try:
        v0 = me.weight_view_tensor(views, 0, cfg, torch.bfloat16)
        v0[:E].normal_().mul_(H ** -0.5)
        me.prefetch(cfg, bufs, views.ptrs, 2)
        del v0
        stream = torch.cuda.current_stream()
        for _ in range(3):
            me.expert_gemm(cfg, bufs, recv, views.ptrs[0], y, stream)
        torch.cuda.synchronize()
        ts = []
        with ClockSampler(local if local is not None else torch.cuda.current_device()) as clk:
            for _ in range(reps):
                flush()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                me.expert_gemm(cfg, bufs, recv, views.ptrs[0], y, stream)
                b.record(stream)
                torch.cuda.synchronize()
                ts.append(a.elapsed_time(b))
        st = me.plan_status(bufs)
        if st[0] != me.STATUS_OK:
            return dict(failed="gemm status %s" % st)
        # context: cuBLAS (torch.matmul) on the same rows, one dense [H, H']
        # weight, same data distribution, timed the same way
        w0 = me.weight_view_tensor(views, 0, cfg, torch.bfloat16)[0].clone()
        for _ in range(3):
            torch.matmul(recv, w0, out=y)
        torch.cuda.synchronize()
        tc = []
        with ClockSampler(local if local is not None else torch.cuda.current_device()) as clk_c:
            for _ in range(reps):
                flush()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                torch.matmul(recv, w0, out=y)
                b.record(stream)
                torch.cuda.synchronize()
                tc.append(a.elapsed_time(b))
        del w0
    finally:
        views.close()
    t = reduce_max([statistics.median(ts)], world)[0]
    t_c = reduce_max([statistics.median(tc)], world)[0]
    flops = 2.0 * P * H * Hp
    tf = flops / (t * 1e-3) / 1e12
    tf_c = flops / (t_c * 1e-3) / 1e12
    burst, sustained, kind = tensor_peaks()
    del recv, y
    torch.cuda.empty_cache()
    name = cfgd["name"].replace("-fp8", "").replace("S%d" % wl.WORKLOADS[base]["S"], "S%d" % cfg.S)
    return dict(workload=name + "-bf16 H'=%d" % Hp, rows=P, rule=rule,
                ms=t, tflops=tf, flops=flops, bound="tensor",
                peak=burst, frac=tf / burst, peak_sustained=sustained,
                frac_sustained=tf / sustained, peak_kind=kind, reps=reps,
                clocks=clk.summary(),
                cublas_same_data=dict(
                    what="torch.matmul of the same rows by one dense [H, H'] weight (no groups), "
                         "same data, same timing; context, not the denominator",
                    ms=t_c, tflops=tf_c, ratio=tf / tf_c, clocks=clk_c.summary()))


def measure_gemm_fp8(me, wl, flush, world, reps=5, S=None, local=None, rule=0):
    """The grouped expert GEMM on the fp8 payload at the fp8 workload's sizes:
    the dispatched e4m3 rows and per-128 scales are widened to bf16 inside the
    GEMM.  Beside it, the unfused route: the identity stand-in writes the
    bf16 rows, then the bf16 GEMM reads them."""
    import torch
    cfgd = wl.cfg_with("fp8", **({"S": S} if S else {}))
    cfg = me.config_from(cfgd, rule)
    cfg16 = me.config_from(dict(cfgd, payload="bf16"), rule)
    idx, _ = wl.routing(cfgd, seed=0)
    bufs = me.PlanBuffers(cfg)
    me.plan(cfg, torch.from_numpy(idx).cuda(), bufs)
    torch.cuda.synchronize()
    st = me.plan_status(bufs)
    if st[0] != me.STATUS_OK:
        return dict(failed="plan status %s (rule %d)" % (st, rule))
    R, E, H, Hp = cfg.R, cfg.E, cfg.H, cfg.Hp
    T, P = R * cfg.S, R * cfg.S * cfg.K
    x = wl.hidden(T, H, seed=1, device="cuda")
    q = torch.empty((P, H), dtype=torch.uint8, device="cuda")
    sc = torch.empty((P, H // 128), dtype=torch.float32, device="cuda")
    me.dispatch(cfg, bufs, x, q, sc)
    del x
    y = torch.empty((P, Hp), dtype=torch.bfloat16, device="cuda")
    stream = torch.cuda.current_stream()

    def timeit(fn):
        for _ in range(2):
            fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(reps):
            flush()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        return reduce_max([statistics.median(ts)], world)[0]

    views = me.WeightViews(cfg, elem_bytes=2)
    try:
        v0 = me.weight_view_tensor(views, 0, cfg, torch.bfloat16)
        v0[:E].normal_().mul_(H ** -0.5)
        me.prefetch(cfg, bufs, views.ptrs, 2)
        del v0
        with ClockSampler(local if local is not None else torch.cuda.current_device()) as clk:
            t_fused = timeit(lambda: me.expert_gemm(cfg, bufs, q, views.ptrs[0], y, stream,
                                                    recv_scale=sc))
        a16 = torch.empty((P, H), dtype=torch.bfloat16, device="cuda")
        t_standin = timeit(lambda: me.expert_standin(cfg, bufs, q, sc, me.EXPERT_IDENTITY, a16,
                                                     stream))
        t_gemm16 = timeit(lambda: me.expert_gemm(cfg16, bufs, a16, views.ptrs[0], y, stream))
        del a16
        st = me.plan_status(bufs)
        if st[0] != me.STATUS_OK:
            return dict(failed="gemm status %s" % st)
    finally:
        views.close()
    flops = 2.0 * P * H * Hp
    burst, sustained, kind = tensor_peaks()
    tf = flops / (t_fused * 1e-3) / 1e12
    del q, sc, y
    torch.cuda.empty_cache()
    name = cfgd["name"].replace("S16384", "S%d" % cfg.S)
    return dict(workload=name + " H'=%d" % Hp, rows=P, rule=rule, ms=t_fused, tflops=tf,
                bound="tensor", peak=burst, frac=tf / burst, peak_sustained=sustained,
                frac_sustained=tf / sustained, peak_kind=kind, reps=reps, clocks=clk.summary(),
                unfused=dict(standin_ms=t_standin, bf16_gemm_ms=t_gemm16,
                             total_ms=t_standin + t_gemm16,
                             what="identity stand-in (fp8 -> bf16 rows in HBM) then the bf16 GEMM"))


def cpu_baseline(cfgd, idx, w, x_dev, rule, budget_s=12.0):
    """The oracle, as it stands, on a bounded sample of the same workload:
    the full plan plus the sampled tokens' dispatch / identity expert /
    combine, sized to about budget_s of one host core, rated over the whole
    workload (value = all picks / the step time the sample stands for)."""
    import numpy as np
    import torch

    from dispatch_moonep_plan_b200 import workloads as wl
    T, P = cfgd["R"] * cfgd["S"], cfgd["R"] * cfgd["S"] * cfgd["K"]
    rng = np.random.default_rng(1)

    def x_rows(tokens):
        return wl.bf16_bits(x_dev[torch.from_numpy(np.asarray(tokens, np.int64)).cuda()])

    n0 = min(256, T)
    t0 = rng.choice(T, n0, replace=False)
    p0 = oracle_sample_step(cfgd, idx, w, x_rows(t0), rule, t0)
    per_tok = (p0["dispatch"] + p0["expert"] + p0["combine"]) / n0
    n = int(max(n0, min(T, (budget_s - p0["plan"]) / max(per_tok, 1e-9))))
    toks = np.sort(rng.choice(T, n, replace=False))
    parts = oracle_sample_step(cfgd, idx, w, x_rows(toks), rule, toks)
    measured, full = oracle_rates(cfgd, parts)
    return dict(kind="oracle", value=P / full, unit=UNIT, cores=1,
                sample="full oracle plan (%d picks, %.3f s) + dispatch/identity expert/combine "
                       "of %d of %d tokens (%.2f s measured), rated over the whole step"
                       % (P, parts["plan"], n, T, measured - parts["plan"]),
                ms_per_full_step=full * 1e3, measured_s=measured,
                parts_s={k: v for k, v in parts.items() if k != "tokens"}, **host_cpu())


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="moonep", choices=["moonep", "reference"])
    ap.add_argument("--workload", default=None,
                    help="the step's workload (default: the largest single-GPU one, hot: R32 "
                         "S8192 E384 K8 H7168 with half of all picks on one expert); with "
                         "--gemm-only the GEMM's routing and sizes (default: the fp8 workload's "
                         "sizes with a bf16 payload)")
    ap.add_argument("--no-sweep", action="store_true",
                    help="leave out the skew sweep and the other workloads' points")
    ap.add_argument("--alpha", type=float, default=None)
    ap.add_argument("--S", type=int, default=None,
                    help="tokens per rank, overriding the workload's (for small profiling cases)")
    ap.add_argument("--rule", type=int, default=0)
    ap.add_argument("--Hp", type=int, default=None,
                    help="with --gemm-only or --side-only: the expert output width H' (default: "
                         "the workload's, else 1536)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-side", action="store_true",
                    help="skip the replica prefetch / grad-reduce measurement")
    ap.add_argument("--gemm-only", action="store_true",
                    help="time only the grouped expert GEMM (--S shrinks it; --workload fp8 takes "
                         "the fp8 payload) and print its line")
    ap.add_argument("--side-only", action="store_true",
                    help="time only the replica prefetch and grad-reduce (fp8 workload's "
                         "routing and weight sizes; --S shrinks the routing) and print their line")
    ap.add_argument("--backward-only", action="store_true",
                    help="time only the backward of combine and of dispatch on --workload "
                         "(--S shrinks it) and print their line")
    ap.add_argument("--plan-only", action="store_true",
                    help="time only the planner on --workload (its inputs and outputs only: "
                         "a few tens of MB on the device) and print its line")
    ap.add_argument("--sweep", default=None,
                    help="also time every workload / skew and write JSON lines to this file")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    from dispatch_moonep_plan_b200 import workloads as wl
    gemm_base = args.workload or "fp8"
    args.payload_fp8 = args.workload == "fp8"  # --gemm-only --workload fp8: the fp8 payload
    if args.workload is None:
        args.workload = "hot"
    cfgd = wl.WORKLOADS[args.workload]
    if args.S is not None:
        cfgd = wl.cfg_with(args.workload, S=args.S, name=cfgd["name"].replace(
            "S%d" % cfgd["S"], "S%d" % args.S))
    if args.impl == "reference":
        run_reference(args, cfgd)
        return
    if args.gemm_only:
        run_gemm_only(args, gemm_base)
        return
    if args.side_only or args.backward_only:
        run_part_only(args, cfgd)
        return
    if args.plan_only:
        run_plan_only(args, cfgd)
        return
    out = run_gpu(args, cfgd)
    if out is not None and int(os.environ.get("WORLD_SIZE", "1")) == 1 and not args.no_sweep:
        out["sweep"] = skew_sweep(args)
        out["other_workloads"] = other_workloads(args)
    if out is not None:
        print(json.dumps(out), flush=True)
    if args.sweep and out is not None:
        run_sweep(args)


def run_plan_only(args, cfgd):
    """The planner alone on the workload's full routing: CUDA events around
    each call (status memset + one cooperative kernel), L2 flushed before
    each outside the events."""
    import torch

    from dispatch_moonep_plan_b200 import moonep as me
    from dispatch_moonep_plan_b200 import workloads as wl
    flush_w = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    cfg = me.config_from(cfgd, args.rule)
    idx, _ = wl.routing(cfgd, seed=0, alpha=args.alpha)
    idx_d = torch.from_numpy(idx).cuda()
    bufs = me.PlanBuffers(cfg)
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        flush_w.zero_()
        me.plan(cfg, idx_d, bufs, stream)
    torch.cuda.synchronize()
    st = me.plan_status(bufs)
    ts = []
    for _ in range(args.steps):
        flush_w.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        me.plan(cfg, idx_d, bufs, stream)
        b.record(stream)
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b) * 1e3)
    # the same call as a node of a CUDA graph, events recorded as graph nodes
    # on both sides (how the planner runs inside the captured step)
    tg = graph_node_times(lambda ev, st: (ev[0].record(st), me.plan(cfg, idx_d, bufs, st),
                                          ev[1].record(st)),
                          2, flush_w.zero_, args, stream)
    print(json.dumps(dict(plan=dict(workload=cfgd["name"], rule=args.rule, status=st,
                                    maxvio=float(bufs.maxvio.item()),
                                    plan_us=statistics.median(ts), mean_us=statistics.mean(ts),
                                    min_us=min(ts), calls=len(ts),
                                    plan_us_in_graph=tg[0] if tg else None))), flush=True)


def run_part_only(args, cfgd):
    """One side measurement on its own (the small ncu cases): the replica
    prefetch and grad-reduce, or the two backward kernels."""
    import torch

    from dispatch_moonep_plan_b200 import moonep as me
    from dispatch_moonep_plan_b200 import workloads as wl
    flush_w = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device="cuda")

    def flush():
        flush_w.zero_()

    if args.side_only:
        print(json.dumps(dict(side=measure_side(me, wl, flush, 1, reps=args.steps, S=args.S,
                                                Hp=args.Hp, rule=args.rule))), flush=True)
        return
    cfg = me.config_from(dict(cfgd, payload="bf16"), args.rule)
    s = me.sizes(cfg)
    T, P, H, K = s.tokens, s.picks, cfg.H, cfg.K
    idx, _ = wl.routing(cfgd, seed=0, alpha=args.alpha)
    bufs = me.PlanBuffers(cfg)
    me.plan(cfg, torch.from_numpy(idx).cuda(), bufs)
    torch.cuda.synchronize()
    st = me.plan_status(bufs)
    if st[0] != me.STATUS_OK:
        raise SystemExit("plan failed with status %s (rule %d)" % (st, args.rule))
    eo = wl.hidden(P, H, seed=3, device="cuda")
    out = measure_backward(me, cfg, bufs, T, P, H, K, flush, 1, eo, reps=args.steps)
    out["workload"] = cfgd["name"]
    print(json.dumps(dict(backward=out)), flush=True)


def run_gemm_only(args, base):
    import torch
    from dispatch_moonep_plan_b200 import moonep as me
    from dispatch_moonep_plan_b200 import workloads as wl
    flush_w = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device="cuda")

    def flush():
        flush_w.zero_()

    if base == "fp8" and args.payload_fp8:
        out = measure_gemm_fp8(me, wl, flush, 1, reps=args.steps, S=args.S, rule=args.rule)
        print(json.dumps(dict(expert_gemm_fp8=out)), flush=True)
        return
    out = measure_gemm(me, wl, flush, 1, reps=args.steps, S=args.S, rule=args.rule, base=base,
                       Hp=args.Hp)
    print(json.dumps(dict(expert_gemm=out)), flush=True)


def _point(out, **extra):
    """The per-workload figures of one run_gpu() result."""
    keys = ("value", "ms_per_step", "maxvio", "plan_us", "dispatch_us", "combine_us",
            "dispatch_GBps", "combine_GBps", "dispatch_frac", "combine_frac", "tokens_per_s",
            "dtype", "clocks")
    d = {k: out[k] for k in keys}
    d["workload"] = out["config"]["workload"]
    d["rule"] = out["config"]["rule"]
    d["routed_rows_per_s"] = d.pop("value")
    d.update(extra)
    return d


def _sub_args(args, alpha, rule):
    a = argparse.Namespace(**vars(args))
    a.alpha, a.rule, a.no_cpu_baseline, a.no_side, a.no_e2e = alpha, rule, True, True, True
    a.steps = min(args.steps, 50)
    a.warm_l2 = False
    return a


def skew_sweep(args):
    """Routed rows/s against maxvio: the Zipf workload (R8 S4096 E256 K8
    H7168 B16) at alpha 0, 0.5, 1.0, 1.5.  Rule 0 where it plans; where it
    needs more than B slots (it fails loudly, as the oracle does) the point
    is taken under rule 1 and the rule-0 failure is recorded beside it."""
    import torch
    from dispatch_moonep_plan_b200 import workloads as wl
    pts = []
    for alpha in wl.WORKLOADS["zipf"]["alphas"]:
        rule0 = None
        for rule in (0, 1):
            try:
                out = run_gpu(_sub_args(args, alpha, rule), wl.WORKLOADS["zipf"], emit=False)
                pts.append(_point(out, alpha=alpha, rule0_failure=rule0))
                break
            except SystemExit as e:
                rule0 = str(e)
            finally:
                torch.cuda.empty_cache()
        else:
            pts.append(dict(alpha=alpha, failed=rule0))
    return pts


def other_workloads(args):
    """The other configurations, one point each: near-uniform routing (R8
    S4096 E64 K6 H2048), the fp8 payload (R16 S16384 E128 K8 H4096, Zipf
    1.2) and the distinct-pick reading of the hot expert."""
    import torch
    from dispatch_moonep_plan_b200 import workloads as wl
    pts = []
    for name in ("uniform", "fp8", "hot_tokens"):
        try:
            out = run_gpu(_sub_args(args, None, 0), wl.WORKLOADS[name], emit=False)
            pts.append(_point(out))
        except SystemExit as e:
            pts.append(dict(workload=name, failed=str(e)))
        torch.cuda.empty_cache()
    return pts


def run_sweep(args):
    """Every workload and skew level, one JSON line each (not the headline)."""
    import torch
    from dispatch_moonep_plan_b200 import workloads as wl
    cases = [("tiny", None, 0), ("tiny-warm", None, 0), ("uniform", None, 0)]
    cases += [("zipf", a, r) for a in (0.0, 0.5, 1.0, 1.5) for r in (0, 1)]
    cases += [("hot", None, 0), ("hot", None, 1), ("hot", None, 2), ("hot_tokens", None, 0),
              ("hot_tokens", None, 1), ("fp8", None, 0), ("fp8", None, 1), ("fp8", None, 2)]
    with open(args.sweep, "w") as f:
        for name, alpha, rule in cases:
            a = argparse.Namespace(**vars(args))
            a.alpha, a.rule, a.no_cpu_baseline, a.no_side, a.no_e2e = alpha, rule, True, True, True
            a.steps = min(args.steps, 50)
            a.warm_l2 = name.endswith("-warm")
            try:
                out = run_gpu(a, wl.WORKLOADS[name.replace("-warm", "")], emit=False)
                if a.warm_l2:
                    out["config"]["l2"] = "warm: no flush between steps (the whole step fits in L2)"
            except SystemExit as e:
                out = dict(workload=name, alpha=alpha, rule=rule, failed=str(e))
            f.write(json.dumps(out) + "\n")
            f.flush()
            torch.cuda.empty_cache()


if __name__ == "__main__":
    main()
