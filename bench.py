#!/usr/bin/env python
"""Decode-attention throughput of the Prism Attention hot path on B200.

One step = one decode step over every layer of the workload: at each
proposal layer the new token's key row is appended and quantized and the
candidate pool is proposed; at every layer the pool is refined and sparse
flash-decode runs over the refined set (the new K/V rows are appended first).
The step is captured once as a CUDA graph and replayed.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config c128k]
    python bench.py --impl reference ...   # the CPU oracle on a bounded sample

Prints one JSON line (rank 0).  Under torchrun every rank runs an independent
replica of the workload (its own sequence, seed = rank): weak scaling, no
collective on the data path; time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from kv_cache_top_proposal_b200 import workload  # noqa: E402

METRIC = "decode attention steps/sec at 128K ctx (all layers); % of HBM roofline"
FALLBACK_HBM_GBS = 6650.0


# --------------------------------------------------------------------------- helpers

def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="c128k", choices=workload.CONFIG_NAMES)
    ap.add_argument("--impl", default="prism", choices=["prism", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="budget of oracle work for the cpu_baseline sample")
    ap.add_argument("--no-cpu", action="store_true", help="skip the cpu_baseline leg")
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--profile-steps", type=int, default=5)
    ap.add_argument("--keys", default="int8", choices=["int8", "int2"],
                    help="proposal key cache: int8 per token (the headline workload) or INT2 per 32-feature group")
    ap.add_argument("--group-agg", default="max", choices=["max", "sum", "mass"],
                    help="how the query heads of a KV head combine into the selection score")
    ap.add_argument("--proposal-select", default="exact", choices=["exact", "quantized"],
                    help="what a proposal layer attends over: its own pool refined with exact scores "
                         "(the default reading) or the top kappa of its quantized scores")
    ap.add_argument("--sets", default="kv_head", choices=["kv_head", "q_head", "sequence"],
                    help="selection granularity: one pool and set per (sequence, KV head), a set per "
                         "query head, or one pool and set per sequence shared by every head")
    ap.add_argument("--grow", action="store_true",
                    help="decode loop over the growing sequence: every replayed step appends one "
                         "token (batch-1 configs); the cache starts short by the replays")
    ap.add_argument("--layers", type=int, default=0,
                    help="keep only the first N layers (small cases for profiling)")
    return ap.parse_args()


def hbm_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            v = float(json.load(f)["hbm_gbs"])
        return v, "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def step_bytes(cfg, keys: str = "int8") -> dict:
    """Algorithmic bytes per op launch (cache reads the method must make)."""
    D, Hkv, T, B = cfg.head_dim, cfg.num_kv_heads, cfg.total_tokens, cfg.batch
    el = 2 if cfg.dtype == "bf16" else 4
    if keys == "int2":
        propose = Hkv * T * (D // 4 + D // 32 * 4)  # 2-bit codes + fp16 (step, zero) per group
    else:
        propose = Hkv * T * (D + 4)  # int8 codes + fp32 scale per (head, position)
    refine = sum(min(cfg.kappa_p, L) for L in cfg.seqlens) * Hkv * D * el
    sparse = sum(min(cfg.kappa, cfg.kappa_p, L) for L in cfg.seqlens) * Hkv * D * el * 2
    dense = Hkv * T * D * el * 2
    # fused refined layer: the pool's key rows once, the selected value rows once
    refine_decode = refine + sparse // 2
    n_prop = len(cfg.proposal_layers)
    return {"propose": propose, "refine": refine, "sparse_decode": sparse, "dense_decode": dense,
            "refine_decode": refine_decode,
            "step": n_prop * propose + cfg.num_layers * refine_decode,
            "step_unfused": n_prop * propose + cfg.num_layers * (refine + sparse),
            "dense_step": cfg.num_layers * dense}


class ClockSampler:
    """SM clock and clock-event reasons of this rank's GPU, sampled by NVML."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, dev_index: int):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._h = None
        try:
            import pynvml

            pynvml.nvmlInit()
            self.nv = pynvml
            props = torch.cuda.get_device_properties(dev_index)
            bus = getattr(props, "pci_bus_id", None)
            try:
                busid = "%08x:%02x:%02x.0" % (getattr(props, "pci_domain_id", 0), bus,
                                              getattr(props, "pci_device_id", 0))
                self._h = pynvml.nvmlDeviceGetHandleByPciBusId(busid.encode())
            except Exception:
                self._h = pynvml.nvmlDeviceGetHandleByIndex(dev_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._h = None

    def _run(self):
        nv = self.nv
        get_r = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons")
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                r = get_r(self._h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            self._stop.wait(0.1)

    def __enter__(self):
        if self._h is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._h is not None:
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


class Dist:
    """One process per GPU.  The ranks share no data: the only collectives
    are the barriers around the timed region and the max over ranks of its
    duration.  `backend` is "nccl" on GPUs; "gloo" serves the CPU tests of
    this host logic."""

    def __init__(self, backend: str = "nccl"):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.backend = backend
        self.pg = None

    def init(self):
        cuda = self.backend == "nccl"
        if cuda:
            torch.cuda.set_device(self.local)
        if self.world > 1:
            import datetime

            import torch.distributed as dist

            kw = {"device_id": torch.device("cuda", self.local)} if cuda else {}
            dist.init_process_group(self.backend, timeout=datetime.timedelta(seconds=120), **kw)
            self.pg = dist

    def barrier(self):
        if self.pg:
            self.pg.barrier()

    def max(self, x: float) -> float:
        if not self.pg:
            return x
        dev = "cuda" if self.backend == "nccl" else "cpu"
        t = torch.tensor([x], dtype=torch.float64, device=dev)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            self.pg.destroy_process_group()


def traffic_for(op: str, workload_name: str, flags: dict):
    """ncu DRAM bytes per launch recorded for this op's kernels, if this run
    launches what was captured: the same workload and flags, and kernel
    sources unchanged since the capture."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        rec = json.load(open(path))[op]
    except Exception:
        return None
    if rec.get("workload") != workload_name or rec.get("flags", {}) != flags:
        return None
    h = hashlib.sha256()
    for f in rec.get("sources", []):
        h.update(open(os.path.join(ROOT, f), "rb").read())
    return rec["dram_bytes_per_launch"] if h.hexdigest() == rec.get("sha256") else None


# --------------------------------------------------------------------------- CPU oracle legs

def unit_list(cfg):
    """The (proposal group, KV head) units of one decode step: a unit is one
    KV head's proposal and every layer of the group that uses its pool."""
    groups = len(cfg.proposal_layers)
    return [(g, h) for h in range(cfg.num_kv_heads) for g in range(groups)]


def unit_bytes(cfg) -> int:
    """Host bytes one prepared unit holds (fp32 K and V of one head, every
    layer of a group)."""
    return cfg.group * 2 * cfg.total_tokens * cfg.head_dim * 4


def unit_inputs(cfg, qs, ks, vs, unit, keys: str = "int8"):
    """Host copies of one unit's inputs and the prefill quantization of its
    key cache (untimed preparation)."""
    import oracle

    grp, h = unit
    G = cfg.G
    lp = grp * cfg.group
    lays = list(range(lp, min(lp + cfg.group, cfg.num_layers)))
    host = {l: (qs[l][:, h * G:(h + 1) * G].float().cpu().numpy(),
                ks[l][h].float().cpu().numpy(), vs[l][h].float().cpu().numpy()) for l in lays}
    quant = oracle.quantize_int2_rows if keys == "int2" else oracle.quantize_rows
    kq, sc = quant(host[lp][1])
    return {"lays": lays, "lp": lp, "host": host, "kq": kq, "sc": sc}


def unit_run(cfg, u, keys: str = "int8", agg: str = "max", proposal_select: str = "exact"):
    """The oracle's work for one unit of a decode step, every sequence: the
    new token's key row quantized, the proposal over the whole sequence, and
    per layer of the group the refine and the attention of every query head."""
    import oracle

    G, D, cu = cfg.G, cfg.head_dim, cfg.cu_seqlens
    scale = float(torch.tensor(1.0 / math.sqrt(D), dtype=torch.float32))
    host, lp, kq, sc = u["host"], u["lp"], u["kq"], u["sc"]
    quant = oracle.quantize_int2_rows if keys == "int2" else oracle.quantize_rows
    for b in range(cfg.batch):
        a, e = cu[b], cu[b + 1]
        if e == a:
            continue
        quant(host[lp][1][e - 1:e])  # the new token's key row
        if keys == "int2":
            pool, ps = oracle.propose_row_int2(host[lp][0][b], kq[a:e], sc[a:e], cfg.kappa_p)
        else:
            pool, ps = oracle.propose_row(host[lp][0][b], kq[a:e], sc[a:e], cfg.kappa_p,
                                          agg="max" if agg == "mass" else agg)
        for l in u["lays"]:
            q, k, v = host[l]
            if l == lp and proposal_select == "quantized":
                idx = oracle.pool_topk(ps, pool, cfg.kappa)
            elif agg == "mass":
                idx, _ = oracle.refine_row_mass(q[b], k[a:e], pool, cfg.kappa, scale)
            else:
                idx, _ = oracle.refine_row(q[b], k[a:e], pool, cfg.kappa, agg=agg)
            for g in range(G):
                oracle.attend(q[b, g], k[a:e], v[a:e], idx, scale)


def oracle_threads(cfg, want: int) -> int:
    """Threads for the oracle: at most the host's cores, the units of a step,
    and what host memory holds (one prepared unit per thread)."""
    n = min(want, len(unit_list(cfg)))
    try:
        import psutil

        n = min(n, max(1, int(0.5 * psutil.virtual_memory().available // unit_bytes(cfg))))
    except Exception:
        pass
    return max(1, n)


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


class OracleRounds:
    """`threads` units of one decode step, prepared once; a round runs each
    of them once, one per thread, and is timed by the wall clock (the C
    oracle releases the interpreter lock while it computes)."""

    def __init__(self, cfg, qs, ks, vs, threads: int, keys: str = "int8", agg: str = "max",
                 proposal_select: str = "exact"):
        from concurrent.futures import ThreadPoolExecutor

        self.cfg, self.keys, self.agg, self.threads = cfg, keys, agg, threads
        self.proposal_select = proposal_select
        self.units = unit_list(cfg)[:threads]
        self.pool = ThreadPoolExecutor(threads)
        self.inputs = list(self.pool.map(lambda u: unit_inputs(cfg, qs, ks, vs, u, keys), self.units))

    def round(self) -> float:
        t0 = time.perf_counter()
        list(self.pool.map(lambda u: unit_run(self.cfg, u, self.keys, self.agg, self.proposal_select),
                           self.inputs))
        return time.perf_counter() - t0

    def close(self):
        self.pool.shutdown()
        self.inputs = None


def oracle_rate(cfg, qs, ks, vs, threads: int, budget_s: float, keys: str = "int8", agg: str = "max",
                proposal_select: str = "exact"):
    """(decode steps/s, units timed, seconds) of the oracle on `threads`
    threads, timed rounds repeated until budget_s seconds."""
    r = OracleRounds(cfg, qs, ks, vs, threads, keys, agg, proposal_select)
    spent, rounds = 0.0, 0
    while spent < budget_s or rounds == 0:
        spent += r.round()
        rounds += 1
    r.close()
    n = rounds * len(r.units)
    return (n / len(unit_list(cfg))) / spent, n, spent


# --------------------------------------------------------------------------- reference arm

def run_reference(args, dist: Dist):
    """The oracle, as it stands, timed on host cores.  A timed step is one
    round: `threads` (proposal group, KV head) units of the decode step, one
    per thread, so ms_per_step is the time of that sample and value is the
    whole-step rate it implies (units/s over units per decode step)."""
    if dist.rank != 0:
        return
    cfg = workload.config(args.config)
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    per_step_units = len(unit_list(cfg))
    threads = oracle_threads(cfg, host_cores())
    # the layers of as many proposal groups as the threads' units need
    n_groups = min(len(cfg.proposal_layers), -(-threads // cfg.num_kv_heads))
    first = list(range(0, min(n_groups * cfg.group, cfg.num_layers)))
    sub = cfg.replace(num_layers=len(first))
    lays = list(workload.generate(cfg, dev, layers=first))
    qs = {x.index: x.q for x in lays}
    ks = {x.index: x.k for x in lays}
    vs = {x.index: x.v for x in lays}
    threads = min(threads, len(unit_list(sub)))
    r = OracleRounds(sub, qs, ks, vs, threads, args.keys, args.group_agg, args.proposal_select)
    del lays, qs, ks, vs
    for _ in range(args.warmup):
        r.round()
    secs = sum(r.round() for _ in range(args.steps))
    n_units = args.steps * len(r.units)
    r.close()
    value = (n_units / per_step_units) / secs
    sample = (f"each timed step = {len(r.units)} of the {per_step_units} (proposal group, KV head) "
              f"units of one {cfg.name} decode step, one per thread on {threads} threads; "
              f"{n_units} units in {secs:.2f} s; value = units/s / {per_step_units}")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "steps/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * secs / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32 selection / f64 attention (CPU oracle)",
        "data": DATA,
        "config": line_config(cfg, args),
        "step_sample": {"units_per_timed_step": len(r.units), "units_per_decode_step": per_step_units,
                        "ms_per_decode_step": 1e3 / value},
        "cpu_baseline": {"value": value, "unit": "steps/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


DATA = "synthetic (seeded drifting-Gaussian RoPE keys, planted salient tokens)"
L2_BYTES = 126 << 20
FLUSH_BYTES = 256 << 20


def needs_flush(nbytes):
    """A step whose distinct bytes are under twice the L2 could be served from it."""
    return nbytes["step"] < 2 * L2_BYTES


def line_config(cfg, args, seqlens0=None, n_grow=0):
    """The `config` object of the JSON line, the same for both arms."""
    nbytes = step_bytes(cfg, args.keys)
    touched = f"a step touches {nbytes['step'] / 1e9:.3f} GB of distinct cache rows (L2 126 MB)"
    return dict(workload_config(cfg),
                l2=(f"L2 flushed between timed steps: each step timed alone, a {FLUSH_BYTES >> 20} MB "
                    f"write between steps outside its event pair; {touched}") if needs_flush(nbytes)
                else f"inputs larger than L2: {touched}",
                refined_layers="fused refine+select+sparse-decode (prism_refine_decode)"
                if args.sets == "kv_head" else "refine and sparse decode (two calls)",
                proposal_select=args.proposal_select, selection_sets=args.sets,
                proposal_keys="int8 per token" if args.keys == "int8"
                else "INT2 per 32-feature group (fp16 step and zero point)",
                graph="one CUDA graph per step",
                group_aggregation=args.group_agg,
                **({"growth": f"decode loop: every replayed step appends one token, "
                              f"from L = {seqlens0[0]} to {seqlens0[0] + n_grow}"}
                   if args.grow and seqlens0 else {}))


def workload_config(cfg):
    return {"workload": f"{cfg.name}: B={cfg.batch}, Hq={cfg.num_q_heads}, Hkv={cfg.num_kv_heads}, "
                        f"d={cfg.head_dim}, L={'ragged' if len(set(cfg.seqlens)) > 1 else cfg.seqlens[0]}, "
                        f"{cfg.num_layers} layers, proposal every {cfg.group}, kappa_p={cfg.kappa_p}, "
                        f"kappa={cfg.kappa}, {cfg.dtype} KV",
            "batch": cfg.batch, "total_tokens": cfg.total_tokens, "layers": cfg.num_layers,
            "kappa_p": cfg.kappa_p, "kappa": cfg.kappa, "parallelism": "replicas (weak)"}


# --------------------------------------------------------------------------- GPU arm

def graph_of(fn, stream):
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fn()
    return g


def run_prism(args, dist: Dist):
    from kv_cache_top_proposal_b200 import prism
    from kv_cache_top_proposal_b200.decoder import PrismDecoder

    dist.init()
    dev = torch.device("cuda", torch.cuda.current_device())
    cfg = workload.config(args.config).replace(seed=dist.rank)
    if args.layers:
        cfg = cfg.replace(num_layers=min(args.layers, cfg.num_layers))
    L = cfg.num_layers
    # ---- cache, queries and the new token rows (generated on the device)
    layers = list(workload.generate(cfg, dev))
    q_all = torch.stack([x.q for x in layers])            # [L][B][Hq][d]
    ks = [x.k for x in layers]
    vs = [x.v for x in layers]
    del layers
    # --grow: a decode loop over one growing sequence; every replay of the step
    # graph appends one token, so it starts short by the number of replays
    n_grow = 1 + 2 * args.warmup + args.steps + max(10, args.steps // 2) if args.grow else 0
    if args.grow and cfg.batch != 1:
        raise SystemExit("--grow decodes one sequence (batch 1)")
    seqlens0 = (cfg.seqlens[0] - n_grow,) if args.grow else cfg.seqlens
    dec = PrismDecoder(seqlens0, cfg.num_q_heads, cfg.num_kv_heads, cfg.head_dim,
                       prism.BF16 if cfg.dtype == "bf16" else prism.F32, L, cfg.group,
                       cfg.kappa_p, cfg.kappa, device=dev, keys=args.keys,
                       capacity=cfg.total_tokens, group_agg=args.group_agg,
                       proposal_select=args.proposal_select, sets=args.sets)
    rows = dec.new_rows.long()
    Hkv = cfg.num_kv_heads
    k_new = torch.stack([k[:, rows].transpose(0, 1).contiguous() for k in ks])  # [L][B][Hkv][d]
    v_new = torch.stack([v[:, rows].transpose(0, 1).contiguous() for v in vs])
    kqs, scs = {}, {}
    for l in cfg.proposal_layers:  # prefill: quantize the whole key cache (untimed)
        if args.keys == "int2":
            Hk, Tk, Dk = ks[l].shape
            kqs[l] = torch.empty((Hk, Tk, Dk // 4), dtype=torch.uint8, device=dev)
            scs[l] = torch.empty((Hk, Tk, Dk // 32, 2), dtype=torch.int16, device=dev)
            prism.quantize_k_int2(dec.p, ks[l], kqs[l], scs[l])
        else:
            kqs[l] = torch.empty(ks[l].shape, dtype=torch.int8, device=dev)
            scs[l] = torch.empty(ks[l].shape[:2], dtype=torch.float32, device=dev)
            prism.quantize_k(dec.p, ks[l], kqs[l], scs[l])
    torch.cuda.synchronize()

    stream = torch.cuda.Stream()
    torch.cuda.set_stream(stream)
    q_layers = [q_all[l] for l in range(L)]

    def step():
        if args.grow:
            dec.advance_on_device(1)
        dec.step(q_layers, ks, vs, kqs, scs, quantize_new=True, k_new=k_new, v_new=v_new)

    step()  # eager once (validates arguments before capture)
    torch.cuda.synchronize()
    status = dec.device_status()
    g = graph_of(step, stream)
    launches = dec.launches_per_step(append=True)

    # a step that touches less than twice the L2 is timed one replay at a time,
    # with a write larger than the L2 between replays, outside the event pairs
    nbytes = step_bytes(cfg, args.keys)
    flush_buf = (torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
                 if needs_flush(nbytes) else None)

    def timed(replay, n, warm):
        for _ in range(warm):
            replay()
        torch.cuda.synchronize()
        dist.barrier()
        torch.cuda.synchronize()
        if flush_buf is None:
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(n):
                replay()
            b.record(stream)
            torch.cuda.synchronize()
            dist.barrier()
            return a.elapsed_time(b) / 1e3  # seconds
        pairs = []
        for i in range(n):
            flush_buf.fill_(i & 0xFF)
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            replay()
            b.record(stream)
            pairs.append((a, b))
        torch.cuda.synchronize()
        dist.barrier()
        return sum(a.elapsed_time(b) for a, b in pairs) / 1e3

    # ---- main timed region (device-resident inputs)
    clk = ClockSampler(torch.cuda.current_device())
    with clk:
        secs = timed(g.replay, args.steps, args.warmup)
    secs = dist.max(secs)
    ms_per_step = secs * 1e3 / args.steps
    value = dist.world * args.steps / secs

    # ---- end to end: pinned host inputs in, outputs out, every step, through
    # PrismDecoder.step_host: one copy per proposal group each way, on a copy
    # stream while the other groups run; one captured graph per step, like
    # the device-resident step
    io = dec.host_io(q_all.dtype)
    for l in range(L):
        io.q_host[l].copy_(q_all[l])
        io.k_new_host[l].copy_(k_new[l])
        io.v_new_host[l].copy_(v_new[l])
    copy_stream = torch.cuda.Stream()

    def e2e_body():
        if args.grow:
            dec.advance_on_device(1)
        dec.step_host(io, ks, vs, kqs, scs, copy_stream, quantize_new=True)

    g_e2e = graph_of(e2e_body, stream)
    e2e_step = g_e2e.replay

    e2e_steps = max(10, args.steps // 2)
    e2e_secs = dist.max(timed(e2e_step, e2e_steps, args.warmup))
    h2d = sum(t.numel() * t.element_size() for t in io.q_host + io.k_new_host + io.v_new_host)
    d2h = io.out_host.numel() * io.out_host.element_size()
    del g_e2e

    if args.grow:
        dec.lengths_from_device()  # the dense comparison sizes its splits from the host copy

    variant = args.sets != "kv_head" or args.proposal_select != "exact" or args.group_agg == "mass"
    if not variant:
        # ---- per-op durations (one graph per op; the queue is filled behind a
        # long memset so every event pair brackets device time only)
        ops = []
        for l in range(L):
            pl = cfg.is_proposal(l)

            def f_prop(l=l):
                if dec.scorer_appends:  # the scorer quantizes the new key rows; the refined layer appends
                    prism.propose_append(dec.p, q_layers[l], k_new[l], kqs[l], scs[l], cfg.kappa_p,
                                         dec.pool[l], dec.pool_cnt[l], dec.ws_prop, sum_group=dec.sum_group)
                    return
                prism.append_kv(dec.p, k_new[l], v_new[l], ks[l], vs[l])
                if args.keys == "int2":
                    prism.quantize_k_int2(dec.p, ks[l], kqs[l], scs[l], tok_rows=dec.new_rows, ws=dec.ws_q)
                    prism.propose_int2(dec.p, q_layers[l], kqs[l], scs[l], cfg.kappa_p, dec.pool[l],
                                       dec.pool_cnt[l], dec.ws_prop)
                else:
                    prism.quantize_k(dec.p, ks[l], kqs[l], scs[l], tok_rows=dec.new_rows, ws=dec.ws_q)
                    prism.propose(dec.p, q_layers[l], kqs[l], scs[l], cfg.kappa_p, dec.pool[l],
                                  dec.pool_cnt[l], dec.ws_prop)

            def f_rd(l=l):
                src = l - l % cfg.group
                # refined layers append their new rows themselves, and so do proposal
                # layers whose scorer took the new key rows
                fa = not cfg.is_proposal(l) or dec.scorer_appends
                prism.refine_decode(dec.p, q_layers[l], ks[l], vs[l], dec.pool[src], dec.pool_cnt[src],
                                    cfg.kappa_p, cfg.kappa, dec.scale, dec.idx[l], dec.cnt[l],
                                    dec.out[l], dec.ws_rd, lse=dec.lse[l],
                                    k_new=k_new[l] if fa else None, v_new=v_new[l] if fa else None,
                                    sum_group=dec.sum_group)

            if pl:
                ops.append(("propose", graph_of(f_prop, stream)))
            ops.append(("refine_decode", graph_of(f_rd, stream)))
        # ~30 MB of memset per queued graph launch keeps the device busy while the
        # host enqueues the profiled sequence
        gate = torch.empty(min(6 << 30, max(256 << 20, len(ops) * (30 << 20))), dtype=torch.uint8,
                           device=dev)
        per_op = {}
        for _ in range(args.profile_steps):
            gate.zero_()
            evs = []
            for name, og in ops:
                a = torch.cuda.Event(enable_timing=True)
                b = torch.cuda.Event(enable_timing=True)
                a.record(stream)
                og.replay()
                b.record(stream)
                evs.append((name, a, b))
            torch.cuda.synchronize()
            for name, a, b in evs:
                per_op.setdefault(name, []).append(a.elapsed_time(b) * 1e3)  # us
        del gate
        per_step_us = {n: sum(v) / args.profile_steps for n, v in per_op.items()}
        dominant = max(per_step_us, key=per_step_us.get)
        iso_us = statistics.mean(per_op[dominant])

        # ---- the dominant kernel as it runs inside the step: every refined-layer
        # launch of the step, in step order with the step's flags (overlapped
        # launches, in-kernel appends), and nothing else; one graph, timed like
        # the step
        def rd_chain():
            for l in range(L):
                pl = cfg.is_proposal(l)
                fa = not pl or dec.scorer_appends
                src = l - l % cfg.group
                prism.refine_decode(dec.p, q_layers[l], ks[l], vs[l], dec.pool[src], dec.pool_cnt[src],
                                    cfg.kappa_p, cfg.kappa, dec.scale, dec.idx[l], dec.cnt[l],
                                    dec.out[l], dec.ws_rd, lse=dec.lse[l],
                                    k_new=k_new[l] if fa else None, v_new=v_new[l] if fa else None,
                                    overlap=dec.fused and not pl and l > 0, sum_group=dec.sum_group)

        g_rd = graph_of(rd_chain, stream)
        rd_reps = max(20, args.steps)
        rd_secs = dist.max(timed(g_rd.replay, rd_reps, args.warmup))
        del g_rd
        instep_us = rd_secs * 1e6 / (rd_reps * L)
        peak, peak_kind = hbm_peak()
        achieved = nbytes["refine_decode"] / (instep_us * 1e-6) / 1e9
        roofline = {"bound": "hbm", "kernel": "refine_decode", "achieved": round(achieved, 1),
                    "peak": peak, "peak_source": peak_kind, "unit": "GB/s",
                    "frac": round(achieved / peak, 4), "traffic": traffic_for("refine_decode", cfg.name,
                                                          {"group_agg": args.group_agg}),
                    "algorithmic_bytes_per_launch": nbytes["refine_decode"],
                    "avg_launch_us": round(instep_us, 3), "launches_per_step": L,
                    "timing": "in step: a graph of the step's refined-layer launches in step order "
                              "with the step's flags, CUDA events on the launching stream, "
                              f"{rd_reps} replays / ({rd_reps} x {L} launches)",
                    "share_of_step": round(L * instep_us / (ms_per_step * 1e3), 3),
                    "isolated_launch_us": round(statistics.mean(per_op["refine_decode"]), 2),
                    "isolated_frac": round(nbytes["refine_decode"]
                                           / (statistics.mean(per_op["refine_decode"]) * 1e-6) / 1e9 / peak, 4),
                    "largest_isolated_op": dominant, "largest_isolated_op_us": round(iso_us, 2)}
        ops_summary = {n: {"us_per_launch": round(statistics.mean(v), 2),
                           "launches_per_step": len(v) // args.profile_steps,
                           "GB/s": round(nbytes[n] / (statistics.mean(v) * 1e-6) / 1e9, 1)}
                       for n, v in per_op.items()}
    else:
        # the variants: the refined (non-proposal) layers of the step, in step
        # order through the layer driver, timed as one graph
        def layer_chain():
            for l in range(L):
                if not cfg.is_proposal(l):
                    dec.layer(l, q_layers[l], ks[l], vs[l], k_new=k_new[l], v_new=v_new[l],
                              overlap=dec.fused and l > 0)

        g_lc = graph_of(layer_chain, stream)
        nref = sum(1 for l in range(L) if not cfg.is_proposal(l))
        reps = max(20, args.steps)
        lc_secs = dist.max(timed(g_lc.replay, reps, args.warmup))
        del g_lc
        per_us = lc_secs * 1e6 / (reps * nref)
        peak, peak_kind = hbm_peak()
        lb = nbytes["refine_decode"] if dec.fused else nbytes["refine"] + nbytes["sparse_decode"]
        achieved = lb / (per_us * 1e-6) / 1e9
        roofline = {"bound": "hbm", "kernel": "refined_layer" if not dec.fused else "refine_decode",
                    "achieved": round(achieved, 1), "peak": peak, "peak_source": peak_kind,
                    "unit": "GB/s", "frac": round(achieved / peak, 4), "traffic": None,
                    "algorithmic_bytes_per_launch": lb, "avg_launch_us": round(per_us, 3),
                    "launches_per_step": nref,
                    "timing": "in step: a graph of the step's refined layers through the layer "
                              f"driver, {reps} replays / ({reps} x {nref} layers)",
                    "share_of_step": round(nref * per_us / (ms_per_step * 1e3), 3)}
        ops_summary = None
    step_achieved = nbytes["step"] / (ms_per_step * 1e-3) / 1e9

    # ---- dense flash-decode over the identical cache (comparison path)
    dense = None
    if not args.no_dense:
        dout = torch.empty_like(dec.out_all)

        def dense_step():
            for l in range(L):
                dec.dense_layer(l, q_layers[l], ks[l], vs[l], dout[l])

        dense_step()
        gd = graph_of(dense_step, stream)
        dn = max(3, args.steps // 10)
        dsecs = dist.max(timed(gd.replay, dn, 2))
        d_ms = dsecs * 1e3 / dn
        dense = {"steps_per_s": round(dist.world * dn / dsecs, 2), "ms_per_step": round(d_ms, 4),
                 "achieved_GBps": round(nbytes["dense_step"] / (d_ms * 1e-3) / 1e9, 1),
                 "sparse_speedup": round(d_ms / ms_per_step, 3)}
        del gd

    status |= dec.device_status()

    # ---- CPU baseline: the oracle on a bounded sample (rank 0, N = 1), on one
    # thread and on as many threads as the host has cores (memory permitting)
    cpu = None
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu:
        units = unit_list(cfg)
        nt = oracle_threads(cfg, host_cores())
        v_n, n_n, s_n = oracle_rate(cfg, q_layers, ks, vs, nt, args.cpu_seconds, args.keys,
                                    args.group_agg, args.proposal_select)
        v_1, n_1, s_1 = oracle_rate(cfg, q_layers, ks, vs, 1, args.cpu_seconds / 3, args.keys,
                                    args.group_agg, args.proposal_select)
        cpu = {"value": v_n, "unit": "steps/s", "cores": nt, "kind": "oracle",
               "sample": f"{n_n} (proposal group, KV head) units of a {cfg.name} decode step "
                         f"({len(units)} per step), {nt} at a time on {nt} threads, "
                         f"{s_n:.1f} s wall; value = units/s / {len(units)}",
               "host_cores": host_cores(),
               "reading": "per (sequence, KV head) sets" if args.sets == "kv_head" else
               "per (sequence, KV head) sets (the oracle's units do not split by the variant's granularity)",
               "single_thread": {"value": v_1, "cores": 1,
                                 "sample": f"{n_1} units on one thread, {s_1:.1f} s"}}

    if dist.rank == 0:
        peak, peak_kind = hbm_peak()
        line = {
            "metric": METRIC, "value": round(value, 3), "unit": "steps/s", "n_gpus": dist.world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": DATA,
            "config": line_config(cfg, args, seqlens0, n_grow),
            "roofline": roofline,
            "step_roofline": {"achieved": round(step_achieved, 1), "peak": peak, "unit": "GB/s",
                              "frac": round(step_achieved / peak, 4),
                              "algorithmic_bytes_per_step": nbytes["step"],
                              "frac_with_unfused_byte_model": round(
                                  nbytes["step_unfused"] / (ms_per_step * 1e-3) / 1e9 / peak, 4),
                              "frac_of_8TBps_nominal": round(step_achieved / 8000.0, 4)},
            "ops": ops_summary,
            "cpu_baseline": cpu,
            "e2e": {"value": round(dist.world * e2e_steps / e2e_secs, 3), "unit": "steps/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": launches * args.steps,
            "gpu_launches_per_step": launches,
            "clocks": clk.summary(),
            "dense": dense,
            "device_status": status,
        }
        print(json.dumps(line), flush=True)
    del g
    dist.close()


def main():
    args = parse()
    dist = Dist()
    if args.impl == "reference":
        run_reference(args, dist)
        return
    run_prism(args, dist)


if __name__ == "__main__":
    main()
