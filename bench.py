"""Benchmark of the CSA / HCA decode path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--config pro]

One step = one decode step of the whole hot path over one batch: for a CSA
layer the state-cache append, the Lightning-indexer scan with top-k and the
sparse attention; for an HCA layer the append and the dense compressed
attention (see compressed_sparse_kv_02_b200.decode: the compression of the
entry a step completes runs on a second stream beside the indexer / the HCA
attention, since no query of the step reads it). The default workload is
the 1M-context Pro-like decode: 8 sequences at position 1,048,575, 128 query
heads sharing a 576-wide latent (d_v = 512), indexer 8 heads x 128, top-1024,
1% planted indexer keys; all inputs synthetic and seeded. The per-step inputs
(about 600 MB of caches read per step) exceed the 126 MB L2, so no flush is
needed between steps.

Prints one JSON line. `value` is decode queries/s from CUDA events around K
replays of a captured CUDA graph of the step (max over ranks); `e2e` is the
same through the C ABI calls with, every step, one host->device copy of the
step's inputs (packed in one pinned buffer) and one device->host copy of its
outputs, the copies of the neighbouring steps overlapping each step's compute
on a second stream (two alternating buffer sets, replayed as one CUDA graph); `roofline` covers the
indexer op (its algorithmic bytes = the visible indexer keys) timed with
events captured around it inside the graph. The default run then adds, under
`secondary`, the metric's other figures from the same GPU: the prefill pass
(65,536 new tokens on 65,536 cached; tokens/s against the sustained bf16
tensor peak) and the mixed-length paged FP8 / FP4 decode (queries/s against
HBM), each with its own roofline, e2e and clock record. `bf16_scores` reports,
outside the timed region, the recall of the indexer's selection on bf16-rounded
scores against its fp32 selection on the same inputs, and both op times.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

METRIC = "CSA/HCA decode queries/s at 1M ctx; HBM GB/s vs peak; prefill tok/s"
UNIT = "queries/s"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1400.0  # sustained under the power cap (earlier measurement on this machine)
EVENT_STEPS = 32  # steps per captured graph
EVENT_STRIDE = 8  # one step in this many carries timing events around its indexer call


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d.get("hbm_gbs", FALLBACK_HBM_GBS)), "measured"
    return FALLBACK_HBM_GBS, "fallback"


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled while the timed region runs."""

    FIELDS = ("index,pci.bus_id,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, period_ms=50):
        self.period_ms = period_ms
        self.proc = None
        self.lines = []
        self.bus = None
        try:
            props = torch.cuda.get_device_properties(torch.cuda.current_device())
            self.bus = "%08X:%02X:%02X.0" % (getattr(props, "pci_domain_id", 0), props.pci_bus_id,
                                             props.pci_device_id)
        except Exception:
            self.bus = None

    def start(self):
        try:
            cmd = ["nvidia-smi", "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                   "-lms", str(self.period_ms)]
            if self.bus:
                cmd += ["-i", self.bus]
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.t.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 10:
                continue
            try:
                sm.append(float(f[2]))
                smax.append(float(f[3]))
            except ValueError:
                continue
            for nm, v in zip(names, f[6:10]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        sm.sort()
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------- workload bytes
def _visible(t, m, n_win):
    return max(0, -(-(t + 1 - n_win) // m))


def bytes_per_query(cfg, ctx_lens=None, n_pairs=1):
    """Algorithmic HBM bytes of one decode query through n_pairs (CSA, HCA) layer pairs, averaged over the
    batch: the visible indexer keys, the attended keys (window rows are bf16, compressed entries in the
    cache's storage type), the append traffic and the query / output I/O."""
    lens = [cfg.ctx] * cfg.batch if ctx_lens is None else list(ctx_lens)
    row = cfg.d_qk * 2  # bf16 raw / window row
    ent = cfg.d_qk * 2 if cfg.kv_dtype == "bf16" else cfg.d_qk + 4  # stored entry (FP8: codes + fp32 scale)
    key_i = cfg.d_idx * 2 if cfg.idx_dtype == "bf16" else cfg.d_idx // 2 + cfg.d_idx // 16
    q_i = cfg.heads_idx * key_i
    tot = {"index": 0.0, "csa_attend": 0.0, "hca_attend": 0.0, "append": 0.0, "io": 0.0}
    for n in lens:
        t = n - 1
        nv, nv_h = _visible(t, cfg.m_csa, cfg.n_win), _visible(t, cfg.m_hca, cfg.n_win)
        n_w = min(cfg.n_win, t + 1)
        tot["index"] += nv * key_i
        tot["csa_attend"] += n_w * row + min(cfg.k, nv) * ent
        tot["hca_attend"] += n_w * row + nv_h * ent
        # appends: the new token's rows (read, written to the ring) and, when a block completes, its m rows
        # of latent + gate logits read back for the fold and one entry written
        app = 2 * (2 * row) + 2 * (2 * cfg.d_idx * 2)
        if (t + 1) % cfg.m_csa == 0:
            app += cfg.m_csa * (2 * row + 2 * cfg.d_idx * 2) + ent + key_i
        if (t + 1) % cfg.m_hca == 0:
            app += cfg.m_hca * 2 * row + ent
        tot["append"] += app
        tot["io"] += 2 * cfg.heads * row + q_i + 2 * cfg.heads * cfg.d_v * 2
    out = {k: int(round(v * n_pairs / len(lens))) for k, v in tot.items()}
    out["total"] = sum(out.values())
    return out


def workload_model(cfg, device="cuda"):
    """The decode model of a workload: uniform lengths and one layer pair, or (mixed) per-sequence
    log-uniform lengths and two layer pairs (CSA, HCA, CSA, HCA)."""
    from compressed_sparse_kv_02_b200 import decode, synth
    if cfg.name == "mixed":
        return decode.DecodeModel(cfg, device=device, ctx_lens=synth.mixed_lengths(cfg), n_pairs=2)
    return decode.DecodeModel(cfg, device=device)


def workload_text(cfg, nq, model):
    if cfg.name == "pro":
        return ("pro-like decode at 1M context: B=%d, t=%d, H=%d, d_qk=%d, d_v=%d, indexer %dx%d, CSA m=4 top-%d, "
                "HCA m'=128, window 128, one CSA + one HCA layer"
                % (nq, cfg.ctx - 1, cfg.heads, cfg.d_qk, cfg.d_v, cfg.heads_idx, cfg.d_idx, cfg.k))
    if cfg.name == "mixed":
        L = model.ctx_lens
        return ("mixed paged decode: B=%d, lengths log-uniform %d..%d (mean %d), H=%d, d_qk=%d, d_v=%d, FP8 e4m3 "
                "KV + fp32 scale per entry, FP4 e2m1 indexer %dx%d with e4m3 scales per 16, top-%d, layers CSA, "
                "HCA, CSA, HCA" % (nq, min(L), max(L), sum(L) // len(L), cfg.heads, cfg.d_qk, cfg.d_v,
                                   cfg.heads_idx, cfg.d_idx, cfg.k))
    return "%s decode: B=%d, t=%d, H=%d, d=%d" % (cfg.name, nq, cfg.ctx - 1, cfg.heads, cfg.d_qk)


# DRAM bytes (read + write) of the indexer op per query, from one ncu capture of its
# kernels on a batch-2 run of the workload, scaled by queries. Each figure is tied to
# the digest of the kernel sources it was captured from; once those sources change
# the figure no longer describes the build and `traffic` is reported as null.
INDEX_OP_SOURCES = ("compressed_sparse_kv_02_b200/csrc/indexer.cu", "compressed_sparse_kv_02_b200/csrc/cskv_device.cuh")
INDEX_OP_DRAM = {  # workload -> (digest of INDEX_OP_SOURCES at the capture, DRAM bytes per query)
    # ncu dram__bytes_read.sum + dram__bytes_write.sum of the scan and the select of one indexer call
    # of the Pro 1M workload at batch 2 (134.31 + 3.74 + 2.20 MB), per query
    "pro": ("929dd11793dc7cb3", 70125568),
}


def sources_digest(paths=INDEX_OP_SOURCES):
    import hashlib
    h = hashlib.sha256()
    for rel in paths:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def index_op_traffic(cfg, nq):
    rec = INDEX_OP_DRAM.get(cfg.name)
    if rec is None or rec[0] != sources_digest():
        return None
    return round(rec[1] * nq)


# ----------------------------------------------------------------- ranks
def rank_config(cfg, rank):
    """Each rank decodes its own batch of sequences: same shapes, its own seed."""
    from compressed_sparse_kv_02_b200 import synth
    return cfg if rank == 0 else synth.Config(**{**cfg.__dict__, "seed": cfg.seed + 17 * rank})


def max_over_ranks(x, device, world):
    """The slowest rank's figure (a MAX all-reduce; every rank gets it)."""
    if world == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank, world, ms_max):
    """Units of all ranks per second of the slowest rank."""
    return units_per_rank * world / (ms_max * 1e-3)


def bf16_peak_sustained():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        if "bf16_tflops_sustained" in d:
            return float(d["bf16_tflops_sustained"]), "measured (sustained)"
    return FALLBACK_BF16_TFLOPS, "fallback"


# ----------------------------------------------------------------- prefill arm
PREFILL_CACHED = 65536
PREFILL_CHUNK = 65536


def run_prefill(args, rank, world):
    """One step = one prefill pass of a 65,536-token chunk onto 65,536 cached tokens through a CSA and an HCA
    layer (compression, indexer + top-k and both attentions for every position of the chunk)."""
    import compressed_sparse_kv_02_b200 as ck
    from compressed_sparse_kv_02_b200 import prefill, synth
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    cfg = rank_config(synth.CONFIGS["prefill"], rank)
    model = prefill.PrefillModel(cfg, cached=PREFILL_CACHED, chunk=PREFILL_CHUNK, device="cuda")
    model.fill_synthetic()
    model.prepare()
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            model.step(stream)
    stream.synchronize()
    if model.check_status() != ck.OK:
        raise RuntimeError("device status after warm-up: %s" % ck.status_string(model.check_status()))
    if world > 1:
        torch.distributed.barrier()
    clocks = ClockSampler()
    clocks.start()
    time.sleep(0.2)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        t0.record(stream)
        for _ in range(args.steps):
            model.step(stream)
        t1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    if world > 1:
        torch.distributed.barrier()
    if model.check_status() != ck.OK:
        raise RuntimeError("device status after the timed region: %s" % ck.status_string(model.check_status()))
    ms_step = max_over_ranks(t0.elapsed_time(t1) / args.steps, dev, world)
    value = whole_job_rate(PREFILL_CHUNK, world, ms_step)
    fl = model.flops()
    peak, src = bf16_peak_sustained()
    achieved = fl["total"] / (ms_step * 1e-3) / 1e12

    # end to end: the chunk's inputs copied in from pinned host memory and the outputs copied out, every pass
    names = ("x", "z", "xi", "zi", "x_h", "z_h", "q", "q_h", "q_idx", "w")
    host = {k_: torch.empty(model.inputs[k_].shape, dtype=model.inputs[k_].dtype, pin_memory=True) for k_ in names}
    for k_ in names:
        host[k_].copy_(model.inputs[k_].cpu())
    outs = (model.idx, model.o_csa, model.o_hca)
    host_out = [torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for o in outs]
    h2d = sum(host[k_].numel() * host[k_].element_size() for k_ in names)
    d2h = sum(o.numel() * o.element_size() for o in outs)
    e2e_steps = 2
    # Within a pass the copies overlap the compute: the chunk's raw rows go in first, then each block's
    # queries on an input stream (the block's calls wait for them), and each block's outputs come back
    # on an output stream as soon as its calls are done (PCIe carries both directions at once). Passes
    # do not overlap each other: a pass starts after the previous one's outputs are out.
    from compressed_sparse_kv_02_b200 import _binding as Bn
    st_c = Bn._stream(stream)
    copy_in, copy_out = torch.cuda.Stream(), torch.cuda.Stream()
    raw = ("x", "z", "xi", "zi", "x_h", "z_h")
    per_block = ("q", "q_h", "q_idx", "w")
    qb = model.q_block
    blocks = [slice(q0, min(PREFILL_CHUNK, q0 + qb)) for q0 in range(0, PREFILL_CHUNK, qb)]
    head, tail = model._calls[:4], model._calls[4 + 3 * len(blocks):]
    body = [model._calls[4 + 3 * i: 7 + 3 * i] for i in range(len(blocks))]

    def e2e_pass():
        start = torch.cuda.Event()
        start.record(stream)
        copy_in.wait_event(start)
        copy_out.wait_event(start)
        ev_raw, ev_in = torch.cuda.Event(), [torch.cuda.Event() for _ in blocks]
        with torch.cuda.stream(copy_in):
            for k_ in raw:
                model.inputs[k_].copy_(host[k_], non_blocking=True)
            ev_raw.record(copy_in)
            for b_, sl in enumerate(blocks):
                for k_ in per_block:
                    model.inputs[k_][sl].copy_(host[k_][sl], non_blocking=True)
                ev_in[b_].record(copy_in)
        stream.wait_event(ev_raw)
        for c in head:
            c(st_c)
        for b_, sl in enumerate(blocks):
            stream.wait_event(ev_in[b_])
            for c in body[b_]:
                c(st_c)
            done = torch.cuda.Event()
            done.record(stream)
            copy_out.wait_event(done)
            with torch.cuda.stream(copy_out):
                for o, ho in zip(outs, host_out):
                    ho[sl].copy_(o[sl], non_blocking=True)
        for c in tail:
            c(st_c)
        out_done = torch.cuda.Event()
        out_done.record(copy_out)
        stream.wait_event(out_done)

    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        e2e_pass()  # warm-up of the copy streams
        e0.record(stream)
        for _ in range(e2e_steps):
            e2e_pass()
        e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, dev, world)
    n_blocks = -(-PREFILL_CHUNK // model.q_block)

    # one more pass, untimed, with events around every call: where the pass's time goes
    from compressed_sparse_kv_02_b200 import _binding as Bn
    st_h = Bn._stream(stream)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in model._calls]
    with torch.cuda.stream(stream):
        for c, (a, b) in zip(model._calls, ev):
            a.record(stream)
            c(st_h)
            b.record(stream)
    torch.cuda.synchronize()
    op_ms = {}
    for c, (a, b) in zip(model._calls, ev):
        op_ms[c.where] = op_ms.get(c.where, 0.0) + a.elapsed_time(b)
    attn_ms = op_ms.get("csa_attend", 0.0) + op_ms.get("hca_attend", 0.0)
    # launches per pass: 4 ring appends + 2 chunk compressions, and per query block the indexer's scan and
    # selection plus one launch per attention call (the query-pair kernel takes calls of at least four
    # queries per SM on the 128-wide latent with 64 heads; the split kernel adds a merge launch)
    n_sm = torch.cuda.get_device_properties(dev).multi_processor_count
    pair = cfg.heads == 64 and cfg.d_qk == 128 and cfg.d_v == 128 and model.q_block >= 4 * n_sm
    per_block = 2 + (2 if pair else 4)
    out = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded Gaussian caches, raw chunk and queries)",
        "config": {
            "workload": "prefill chunk: %d new tokens on %d cached (one sequence), H=%d, d=%d (K=V), indexer "
                        "%dx%d, CSA m=4 top-%d, HCA m'=128, window 128, one CSA + one HCA layer"
                        % (PREFILL_CHUNK, PREFILL_CACHED, cfg.heads, cfg.d_qk, cfg.heads_idx, cfg.d_idx, cfg.k),
            "config_name": cfg.name,
            "parallelism": "replicas" if world == 1 else "dp%d (independent sequences per GPU)" % world,
            "l2": "inputs larger than L2 (queries alone %.0f MB)" % (2 * model.inputs["q"].numel() * 2 / 1e6),
            "timing": "%d eager passes between CUDA events on the launching stream" % args.steps,
        },
        "clocks": {"sm_mhz": clk["sm_mhz"], "sm_max_mhz": clk["sm_max_mhz"], "reasons": clk["reasons"],
                   "samples": clk["samples"]},
        "roofline": {
            "bound": "tensor",
            "kernel": "whole prefill pass (indexer scan + top-k + CSA and HCA attention)",
            "achieved": round(achieved, 1),
            "peak": peak,
            "peak_source": src,
            "unit": "TFLOP/s",
            "frac": round(achieved / peak, 4),
            "traffic": None,
            "algorithmic_flops_per_step": fl,
        },
        "e2e": {"value": round(whole_job_rate(PREFILL_CHUNK, world, e2e_ms), 2), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps},
        "gpu_launches": (6 + per_block * n_blocks) * args.steps,
        "op_ms_untimed_breakdown": {k_: round(v_, 3) for k_, v_ in op_ms.items()},
        "attention_tflops_untimed": round((fl["csa_attend"] + fl["hca_attend"]) / (attn_ms * 1e-3) / 1e12, 1)
        if attn_ms > 0 else None,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = prefill_cpu_baseline(model, cfg, budget_s=args.cpu_budget)
    return out


def prefill_cpu_baseline(model, cfg, budget_s=20.0):
    """The oracle on sampled chunk positions (window rows from the chunk), scaled to tokens/s."""
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import oracle
    from gpu_helpers import layer_entries, stored_bf16
    oracle.build()
    cores = os.cpu_count() or 1
    oracle.set_threads(cores)
    csa, hca = model.layers
    inp, c0 = model.inputs, model.cached
    sm = 1.0 / math.sqrt(cfg.d_qk)
    g = torch.Generator().manual_seed(cfg.seed)
    pos = [c0 + 127, c0 + model.chunk - 1] + torch.randint(c0 + 128, c0 + model.chunk - 1, (4096,),
                                                             generator=g).tolist()
    ent = layer_entries(csa, 0, oracle.visible_entries(c0 + model.chunk - 1, cfg.m_csa, cfg.n_win))
    ent_h = layer_entries(hca, 0, oracle.visible_entries(c0 + model.chunk - 1, cfg.m_hca, cfg.n_win))["kv"]
    done, t_cpu = 0, 0.0
    for t in pos:
        if t_cpu >= budget_s:
            break
        i = t - c0
        nv = oracle.visible_entries(t, cfg.m_csa, cfg.n_win)
        nvh = oracle.visible_entries(t, cfg.m_hca, cfg.n_win)
        win = stored_bf16(inp["x"][0, max(0, i - 127):i + 1])
        win_h = stored_bf16(inp["x_h"][0, max(0, i - 127):i + 1])
        if i < 127:
            continue  # keep the sample to positions whose window lies inside the chunk
        x = dict(q=stored_bf16(inp["q"][i]), qi=stored_bf16(inp["q_idx"][i]), w=inp["w"][i].double().cpu().numpy(),
                 kv=ent["kv"].rows_subset(0, nv), ki=ent["idx"].rows_subset(0, nv), kvh=ent_h.rows_subset(0, nvh),
                 qh=stored_bf16(inp["q_h"][i]))
        t0 = time.perf_counter()
        oracle.csa_query(t, cfg.m_csa, cfg.n_win, cfg.k, x["q"], x["qi"], x["w"], win, x["kv"], x["ki"], cfg.d_v, sm)
        oracle.hca_query(t, cfg.m_hca, cfg.n_win, x["qh"], win_h, x["kvh"], cfg.d_v, sm)
        t_cpu += time.perf_counter() - t0
        done += 1
    return {"value": round(done / t_cpu, 4), "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": "%d sampled chunk positions (indexer + top-k + CSA and HCA attention per position, fp64; "
                      "compression not timed), %.1f s of host time, extrapolated to tokens/s" % (done, t_cpu)}


# ----------------------------------------------------------------- our arm
def run_ours(args, rank, world):
    import compressed_sparse_kv_02_b200 as ck
    from compressed_sparse_kv_02_b200 import decode, synth
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    cfg = synth.CONFIGS[args.config]
    if args.batch:
        cfg = synth.Config(**{**cfg.__dict__, "batch": args.batch})
    cfg = rank_config(cfg, rank)
    model = workload_model(cfg)
    model.fill_synthetic()
    model.prepare()
    stream = torch.cuda.Stream()
    nq = cfg.batch

    # eager warm-up (also loads the kernels), then the status word must be clean
    with torch.cuda.stream(stream):
        for _ in range(max(1, args.warmup)):
            model.step(stream)
    stream.synchronize()
    st = model.check_status()
    if st != ck.OK:
        raise RuntimeError("device status after warm-up: %s" % ck.status_string(st))

    # The timed graph holds n_ev steps with timing events around each step's indexer call; a second graph
    # holds the remaining K mod n_ev steps, so that exactly K steps are timed. A third graph (not timed)
    # records events around every call, for the per-op breakdown.
    calls, ops = model._calls, model._ops
    idx_i = [i for i, c in enumerate(calls) if c.where == "csa_index_score_topk"][0]
    n_ev = min(EVENT_STEPS, max(1, args.steps))
    reps, rem = divmod(args.steps, n_ev)
    mk = lambda: (torch.cuda.Event(enable_timing=True, external=True), torch.cuda.Event(enable_timing=True, external=True))
    ev = [mk() for _ in range(n_ev)]
    evb = [[mk() for _ in calls] for _ in range(n_ev)]
    s = ck._binding._stream(stream)
    graph = torch.cuda.CUDAGraph()
    # Timing events sit around the indexer call of every EVENT_STRIDE-th step only: an event between
    # two kernels keeps the second from starting early (programmatic dependent launch), so events in
    # every step would slow the step they measure.
    ev_steps = [j for j in range(n_ev) if j % EVENT_STRIDE == EVENT_STRIDE - 1] or [n_ev - 1]
    with torch.cuda.graph(graph, stream=stream):
        for j in range(n_ev):
            if j in ev_steps:  # the indexer runs on the step's main stream
                model.run(ops, stream, lambda i, c, st, j=j: ev[j][0].record(st) if i == idx_i else None,
                          lambda i, c, st, j=j: ev[j][1].record(st) if i == idx_i else None)
            else:
                model.run(ops, stream)
    graph_rem = None
    if rem:
        graph_rem = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph_rem, stream=stream):
            for _ in range(rem):
                model.run(ops, stream)
    graph_b = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph_b, stream=stream):
        for j in range(n_ev):  # events on the stream each call runs on (side-stream calls overlap the others)
            model.run(ops, stream, lambda i, c, st, j=j: evb[j][i][0].record(st),
                      lambda i, c, st, j=j: evb[j][i][1].record(st))
    # graphs replay on the stream the timing events are recorded on
    with torch.cuda.stream(stream):
        for _ in range(max(1, -(-args.warmup // n_ev))):
            graph.replay()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clocks = ClockSampler()
    clocks.start()
    time.sleep(0.2)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        t0.record(stream)
        for _ in range(reps):
            graph.replay()
        if graph_rem is not None:
            graph_rem.replay()
        t1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    if world > 1:
        torch.distributed.barrier()
    steps_timed = args.steps
    ms_total = t0.elapsed_time(t1)
    idx_vals = [ev[j][0].elapsed_time(ev[j][1]) for j in ev_steps] if reps else []
    with torch.cuda.stream(stream):
        graph_b.replay()
    torch.cuda.synchronize()
    op_ms = {}
    for i, c in enumerate(calls):
        vals = [evb[j][i][0].elapsed_time(evb[j][i][1]) for j in range(n_ev)]
        op_ms["%s#%d" % (c.where, i)] = round(sum(vals) / len(vals), 5)
    idx_ms_avg = sum(idx_vals) / len(idx_vals) if idx_vals else op_ms["csa_index_score_topk#%d" % idx_i]
    st = model.check_status()
    if st != ck.OK:
        raise RuntimeError("device status after the timed region: %s" % ck.status_string(st))
    ms_step = max_over_ranks(ms_total / steps_timed, dev, world)
    value = whole_job_rate(nq, world, ms_step)

    # end to end: every step copies its inputs in from pinned host memory and its outputs (both layers'
    # attention outputs) out. A step's input tensors are views of one contiguous device buffer (its outputs
    # of another), mirrored by one pinned host buffer each, so a step is one copy in, the step's calls
    # through the C ABI, one copy out. Two such buffer sets alternate, and the copies run on a second
    # stream while the other set's step computes (as a serving loop pipelines them): while step A runs,
    # B's inputs are copied in and B's previous outputs out; while B runs, A's outputs out and A's next
    # inputs in. Two steps (copies and calls) are captured in one CUDA graph and replayed.
    def flat_offsets(items):
        offs, off = [], 0
        for v in items:
            offs.append(off)
            off += (v.numel() * v.element_size() + 255) // 256 * 256
        return offs, off
    in_items = [(li, k_) for li, d in model.inputs.items() for k_ in d]
    in_offs, in_bytes = flat_offsets([model.inputs[li][k_] for li, k_ in in_items])
    out_items = [(li, n) for li in model.out for n in ("o_csa", "o_hca")]
    out_offs, out_bytes = flat_offsets([model.out[li][n] for li, n in out_items])
    src_in = {key: model.inputs[key[0]][key[1]] for key in in_items}
    out_proto = {key: model.out[key[0]][key[1]] for key in out_items}
    sets = []
    for _ in range(2):
        dev_in = torch.empty(in_bytes, dtype=torch.uint8, device=dev)
        host_in = torch.zeros(in_bytes, dtype=torch.uint8, pin_memory=True)
        dev_out = torch.empty(out_bytes, dtype=torch.uint8, device=dev)
        host_out = torch.empty(out_bytes, dtype=torch.uint8, pin_memory=True)
        for key, off in zip(in_items, in_offs):
            v = src_in[key]
            nb = v.numel() * v.element_size()
            view = dev_in[off:off + nb].view(v.dtype).view(v.shape)
            view.copy_(v)
            host_in[off:off + nb].copy_(v.contiguous().view(-1).view(torch.uint8).cpu())
            model.inputs[key[0]][key[1]] = view
        for key, off in zip(out_items, out_offs):
            o = out_proto[key]
            model.out[key[0]][key[1]] = dev_out[off:off + o.numel() * o.element_size()].view(o.dtype).view(o.shape)
        ops_set = list(model.prepare())
        sets.append((dev_in, host_in, dev_out, host_out, ops_set, model._keep))
    h2d, d2h = in_bytes, out_bytes
    e2e_steps = 2 * max(1, min(args.steps, 200) // 2)
    copy_stream = torch.cuda.Stream()

    def run_calls(ops_set):
        model.run(ops_set, stream)

    def two_steps():
        (inA, hinA, outA, houtA, cA, _), (inB, hinB, outB, houtB, cB, _) = sets
        ev = [torch.cuda.Event() for _ in range(4)]
        ev[0].record(stream)
        copy_stream.wait_event(ev[0])
        with torch.cuda.stream(copy_stream):
            inB.copy_(hinB, non_blocking=True)      # B's inputs for this replay's second step
            houtB.copy_(outB, non_blocking=True)    # B's outputs of the previous replay
        ev[1].record(copy_stream)
        run_calls(cA)                               # step A on its inputs (copied in last replay)
        ev[2].record(stream)
        copy_stream.wait_event(ev[2])
        with torch.cuda.stream(copy_stream):
            houtA.copy_(outA, non_blocking=True)    # A's outputs
            inA.copy_(hinA, non_blocking=True)      # A's inputs for the next replay
        stream.wait_event(ev[1])
        run_calls(cB)                               # step B
        ev[3].record(copy_stream)
        stream.wait_event(ev[3])

    with torch.cuda.stream(stream):
        for st_ in sets:  # both sets' inputs in place, once
            st_[0].copy_(st_[1], non_blocking=True)
        for _ in range(max(1, args.warmup)):
            two_steps()
    stream.synchronize()
    e2e_graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(e2e_graph, stream=stream):
        two_steps()
    with torch.cuda.stream(stream):
        e2e_graph.replay()
        stream.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(e2e_steps // 2):
            e2e_graph.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, dev, world)
    del e2e_graph
    st = model.check_status()
    if st != ck.OK:
        raise RuntimeError("device status after the end-to-end steps: %s" % ck.status_string(st))

    bq = bytes_per_query(cfg, model.ctx_lens, model.n_pairs)
    hbm, src = peaks()
    idx_bytes = bq["index"] * nq // model.n_pairs  # one indexer call (the first CSA layer's)
    achieved = idx_bytes / (idx_ms_avg * 1e-3) / 1e9
    path_gbs = bq["total"] * nq / (ms_step * 1e-3) / 1e9
    kernels_per_step = 0
    for c in calls:
        kernels_per_step += {"cskv_cache_append": 1, "cskv_cache_append_ring": 1, "cskv_cache_append_emit": 1,
                             "csa_index_score_topk": 2, "csa_attend": 2, "hca_attend": 2}[c.where]
    out = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": UNIT,
        "n_gpus": world,
        "steps": steps_timed,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if cfg.kv_dtype == "bf16" else "fp8 KV / fp4 indexer",
        "data": "synthetic (seeded Gaussian caches%s)" % (", 1% planted indexer keys" if cfg.planted_frac else
                                                           ", random FP8 / FP4 codes" if cfg.kv_dtype != "bf16" else ""),
        "config": {
            "workload": workload_text(cfg, nq, model),
            "config_name": cfg.name,
            "batch_per_gpu": nq,
            "context": max(model.ctx_lens),
            "parallelism": "replicas" if world == 1 else "dp%d (independent sequences per GPU)" % world,
            "l2": "inputs larger than L2 (%.0f MB read per step)" % (bq["total"] * nq / 1e6),
            "timing": "CUDA graph of %d steps replayed %d times (+%d); CUDA events on the launching stream; "
                      "the indexer op timed in one step of %d" % (n_ev, reps, rem, EVENT_STRIDE),
        },
        "clocks": {"sm_mhz": clk["sm_mhz"], "sm_max_mhz": clk["sm_max_mhz"], "reasons": clk["reasons"],
                   "samples": clk["samples"]},
        "roofline": {
            "bound": "hbm",
            "kernel": "csa_index_score_topk (indexer scan + top-k select)",
            "achieved": round(achieved, 1),
            "peak": hbm,
            "peak_source": src,
            "unit": "GB/s",
            "frac": round(achieved / hbm, 4),
            "traffic": index_op_traffic(cfg, nq),
            "algorithmic_bytes_per_launch": idx_bytes,
            "avg_launch_ms": round(idx_ms_avg, 5),
        },
        "op_ms_untimed_breakdown": op_ms,
        "path_roofline": {
            "bound": "hbm", "achieved": round(path_gbs, 1), "peak": hbm, "unit": "GB/s",
            "frac": round(path_gbs / hbm, 4), "bytes_per_query": bq,
        },
        "e2e": {"value": round(whole_job_rate(nq, world, e2e_ms), 2), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps},
        "gpu_launches": kernels_per_step * steps_timed,
    }
    if rank == 0:
        out["bf16_scores"] = bf16_score_report(model, cfg, stream)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(model, cfg, budget_s=args.cpu_budget)
    return out


def bf16_score_report(model, cfg, stream, reps: int = 20) -> dict:
    """The indexer's selection mode on bf16-rounded scores (DeepSeek-V4 report digest, section 7: index
    scores in BF16) against the fp32 selection, on the first CSA layer of the step's own inputs (after the
    timed region): the recall |S_bf16 & S_fp32| / |S_fp32| averaged over the queries, and the op time of
    each mode (CUDA events on the launching stream, mean of `reps` calls)."""
    import compressed_sparse_kv_02_b200 as ck
    layer, inp = model.layers[0], model.inputs[0]
    nq, k = cfg.batch, cfg.k
    res = {}
    for bf16 in (False, True):
        idx = torch.empty(nq, k, dtype=torch.int32, device="cuda")
        cnt = torch.empty(nq, dtype=torch.int32, device="cuda")
        ws = torch.empty(ck.csa_index_ws_bytes(layer, nq, cfg.heads_idx, model.max_pos, k), dtype=torch.uint8,
                         device="cuda")

        def call():
            ck.csa_index_score_topk(layer, model.seq, model.pos, model.max_pos, inp["q_idx"], inp["w"], k, idx, cnt,
                                    q_idx_scale=inp.get("q_idx_scale"), workspace=ws, status=model.status,
                                    stream=stream, score_bf16=bf16)
        with torch.cuda.stream(stream):
            call()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(reps):
                call()
            e1.record(stream)
        stream.synchronize()
        res[bf16] = (idx.cpu().numpy(), cnt.cpu().numpy(), e0.elapsed_time(e1) / reps)
    (i32, c32, t32), (i16, c16, t16) = res[False], res[True]
    rec = [len(set(i16[b, :c16[b]].tolist()) & set(i32[b, :c32[b]].tolist())) / max(1, int(c32[b]))
           for b in range(nq)]
    return {"recall_vs_fp32": round(float(np.mean(rec)), 5), "recall_min": round(float(np.min(rec)), 5),
            "index_op_ms_fp32": round(t32, 5), "index_op_ms_bf16": round(t16, 5),
            "note": "scores rounded to bf16 (RNE) before the selection; the scan reads the same keys, so the op "
                    "time does not change"}


# ----------------------------------------------------------------- the oracle on host cores
def _window_rows(layer, new_x, b, t):
    """Raw window rows of positions t-n_win+1 .. t in position order, from the synthesised state: the
    ring slots of positions t-n_win+1 .. t-1 (written by the synthesis, never by a decode step, which only
    writes the slot of t) and the decode token's own row."""
    from gpu_helpers import stored_bf16
    ws = max(0, t - layer.n_win + 1)
    slots = [p % layer.n_win for p in range(ws, t)]
    rows = torch.cat([layer.ring_x[b][slots], new_x[b].reshape(1, -1).to(layer.ring_x.dtype)], 0)
    return stored_bf16(rows)


def _oracle_inputs(model, cfg, b):
    """Host copies (oracle storage views) of sequence b's synthesised caches and query."""
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import oracle
    from gpu_helpers import layer_entries, stored_bf16, stored_fp4
    t = model.ctx_lens[b] - 1
    csa, hca = model.layers[0], model.layers[1]
    nv = oracle.visible_entries(t, cfg.m_csa, cfg.n_win)
    nv_h = oracle.visible_entries(t, cfg.m_hca, cfg.n_win)
    ent = layer_entries(csa, b, nv)
    inp = model.inputs[0]
    qi = (stored_bf16(inp["q_idx"][b]) if cfg.idx_dtype == "bf16" else
          stored_fp4(inp["q_idx"][b], inp["q_idx_scale"][b]))
    return dict(t=t, win=_window_rows(csa, inp["csa_x"], b, t), kv=ent["kv"], ki=ent["idx"],
                q=stored_bf16(inp["q_csa"][b]), qi=qi, w=inp["w"][b].double().cpu().numpy(),
                win_h=_window_rows(hca, inp["hca_x"], b, t), kv_h=layer_entries(hca, b, nv_h)["kv"],
                q_h=stored_bf16(inp["q_hca"][b]))


def _oracle_query(cfg, x):
    import oracle
    sm = 1.0 / math.sqrt(cfg.d_qk)
    oracle.csa_query(x["t"], cfg.m_csa, cfg.n_win, cfg.k, x["q"], x["qi"], x["w"], x["win"], x["kv"], x["ki"],
                     cfg.d_v, sm)
    oracle.hca_query(x["t"], cfg.m_hca, cfg.n_win, x["q_h"], x["win_h"], x["kv_h"], cfg.d_v, sm)


def cpu_baseline(model, cfg, budget_s=20.0):
    import oracle
    oracle.build()
    cores = os.cpu_count() or 1
    oracle.set_threads(cores)
    done, t_cpu = 0, 0.0
    xs = [_oracle_inputs(model, cfg, b) for b in range(min(2, cfg.batch))]
    # a query goes through n_pairs layer pairs; the sample runs the first pair and charges n_pairs of it
    while t_cpu < budget_s and done < 4 * cfg.batch:
        x = xs[done % len(xs)]
        t0 = time.perf_counter()
        _oracle_query(cfg, x)
        t_cpu += (time.perf_counter() - t0) * model.n_pairs
        done += 1
    return {"value": round(done / t_cpu, 4), "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": "%d full decode queries (CSA indexer+top-k+attention and HCA attention, fp64, %d layer "
                      "pair(s)) of the same workload, %.1f s of host time" % (done, model.n_pairs, t_cpu)}


def run_reference(args, rank, world):
    """The oracle as the reference arm: K steps, each a bounded sample of the decode workload. The caches,
    rings and queries are synthesised on the GPU by torch's generators (no decode step runs: the oracle
    reads the synthesised state, with the decode token's own row as the newest window row)."""
    from compressed_sparse_kv_02_b200 import synth
    import oracle
    oracle.build()
    cfg = synth.CONFIGS[args.config]
    model = workload_model(cfg)
    model.fill_synthetic()
    torch.cuda.synchronize()
    cores = os.cpu_count() or 1
    oracle.set_threads(cores)
    xs = [_oracle_inputs(model, cfg, b) for b in range(min(cfg.batch, 2))]
    # calibrate one query; a step is one query when K of them fit in ~3 minutes, else a head/entry sample
    t0 = time.perf_counter()
    _oracle_query(cfg, xs[0])
    t_q = time.perf_counter() - t0
    frac = min(1.0, 180.0 / max(1e-9, t_q * (args.steps + args.warmup)))
    sample = xs
    if frac < 1.0:
        sample = []
        for x in xs:
            y = dict(x)
            nv = x["ki"].rows
            n_sub = max(cfg.k + 1, int(nv * frac))
            h_sub = max(1, int(cfg.heads * frac))
            y["ki"] = x["ki"].rows_subset(0, n_sub)
            y["kv"] = x["kv"].rows_subset(0, n_sub)
            y["q"] = x["q"].rows_subset(0, h_sub)
            y["q_h"] = x["q_h"].rows_subset(0, h_sub)
            y["t"] = n_sub * cfg.m_csa + cfg.n_win - 1
            nvh = oracle.visible_entries(y["t"], cfg.m_hca, cfg.n_win)
            y["kv_h"] = x["kv_h"].rows_subset(0, nvh)
            sample.append(y)
    for i in range(args.warmup):
        _oracle_query(cfg, sample[i % len(sample)])
    t0 = time.perf_counter()
    for i in range(args.steps):
        _oracle_query(cfg, sample[i % len(sample)])
    dt = (time.perf_counter() - t0) / max(1, args.steps)
    value = frac / dt
    desc = ("one full decode query per step" if frac >= 1.0 else
            "per step a %.4f sample of one decode query (first entries of the indexer scan, first heads of "
            "the attention), scaled to queries/s" % frac)
    return {
        "metric": METRIC, "impl": "reference", "value": round(value, 4), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": cfg.name, "config_name": cfg.name},
        "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def secondary_workloads(args, rank, world):
    """The metric's other two figures, measured in the same run on the same GPU after the headline decode:
    the prefill pass (tokens/s against the sustained bf16 tensor peak) and the mixed-length paged FP8 / FP4
    decode (queries/s against HBM). Each keeps its own roofline, e2e and clock record; the oracle is not
    run for them here (`--config prefill` / `--config mixed` give their full lines with a cpu_baseline)."""
    import copy
    out = {}
    for name, steps in (("prefill", 6), ("mixed", 64)):
        a = copy.copy(args)
        a.config, a.steps, a.warmup, a.no_cpu_baseline, a.batch = name, steps, 3, True, 0
        torch.cuda.empty_cache()
        r = run_prefill(a, rank, world) if name == "prefill" else run_ours(a, rank, world)
        keep = ("value", "unit", "ms_per_step", "steps", "warmup", "dtype", "config", "clocks", "roofline", "e2e",
                "gpu_launches", "op_ms_untimed_breakdown", "path_roofline", "attention_tflops_untimed")
        out[name] = {k: r[k] for k in keep if k in r}
        torch.cuda.synchronize()
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2048)
    ap.add_argument("--warmup", type=int, default=8)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default="pro")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=20.0)
    ap.add_argument("--batch", type=int, default=0, help="override the workload's batch (profiling captures)")
    ap.add_argument("--no-secondary", action="store_true",
                    help="skip the prefill and mixed-workload figures that the default (pro) run adds")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":  # the oracle runs on rank 0's host cores only; no process group
        if rank == 0:
            torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
            print(json.dumps(run_reference(args, rank, world)), flush=True)
        return
    if world > 1:
        import datetime
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        out = run_prefill(args, rank, world) if args.config == "prefill" else run_ours(args, rank, world)
        if args.config == "pro" and not args.no_secondary:
            out["secondary"] = secondary_workloads(args, rank, world)
        if rank == 0:
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
