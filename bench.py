#!/usr/bin/env python
"""Benchmark of the MSA hot path (index select + sparse attention) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step is one pass of the whole path over one batch: msa_index_select
(index scores with the fused causal block max pool, then top-k) followed by
msa_sparse_attn on its ids, with inputs resident in HBM.  Decode workloads
report algorithmic HBM GB/s (K_idx read once, the selected K/V blocks, q,
q_idx and the output; scores, ids and partials are overhead, not credit);
prefill workloads report effective TFLOP/s (2*d_idx per visible (query, group,
key) for the index GEMM plus 4*d per selected visible (query head, key)).

Multi-GPU (torchrun): every rank runs its own replica of the workload (weak
scaling, no collective on the data path); the step time is the max over ranks.
--impl reference runs the float64 CPU oracle on a bounded sample of the same
workload on rank 0 (the other ranks exit).
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

from block_sparse_gqa_03_b200.inputs import WORKLOADS, make_inputs  # noqa: E402

METRIC = "MSA decode µs/step & HBM GB/s at 128K–1M ctx; prefill effective TFLOP/s"
DEFAULT_WORKLOAD = "decode_128k"
L2_BYTES = 126 * 2**20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# Per-launch DRAM traffic (read + write bytes) of a kernel, from one ncu capture
# at batch 4 scaled by 4 to the workload's batch of 16 (the work grows in
# proportion).  An entry is removed when its kernel changes; absent entries
# report null.
TRAFFIC = {
    ("decode_128k", "attn"): 4 * (134.483968e6 + 3.917824e6),
    ("decode_128k", "scan"): 4 * (134.275584e6 + 4.156672e6),
}
L2_FLUSH_BYTES = 256 * 2**20


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if args.impl == "ours" else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available() and args.impl == "ours":
        torch.cuda.set_device(0)
    return world, rank, local


def max_over_ranks(x: float, world: int) -> float:
    """The largest of the ranks' values (step times are reported as the slowest rank's)."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ----------------------------------------------------------------- work counts
def positions(prob, seq_lens, device):
    L = (torch.full((prob.batch,), prob.max_kv, device=device, dtype=torch.int64)
         if seq_lens is None else seq_lens.to(torch.int64))
    t = torch.arange(prob.n_q, device=device, dtype=torch.int64)
    p = L[:, None] - prob.n_q + t[None, :]
    lim = torch.minimum(L[:, None], p + 1) if prob.causal else L[:, None].expand(-1, prob.n_q)
    return L, lim.clamp(min=0)  # lim[b, t]: visible tokens are j < lim


def selected_visible_tokens(prob, ids, lim):
    """Visible tokens in the selected blocks, per (b, t, g): [b, n_q, h] int64."""
    idl = ids.to(torch.int64)
    start = idl * prob.block
    n = (lim[:, :, None, None] - start).clamp(min=0, max=prob.block)
    n = torch.where(idl >= 0, n, torch.zeros_like(n))
    return n.sum(-1)


def work_units(prob, x, ids):
    """Algorithmic bytes (decode) or flops (prefill), split by stage."""
    L, lim = positions(prob, x["seq_lens"], ids.device)
    sel_tok = selected_visible_tokens(prob, ids, lim)  # [b, n_q, h]
    if prob.is_decode:
        kidx = int(L.sum()) * prob.d_idx * 2
        qidx = prob.batch * prob.n_q * prob.h * prob.d_idx * 2
        kv = int(sel_tok.sum()) * prob.d * 2 * 2
        q_o = 2 * prob.batch * prob.n_q * prob.H * prob.d * 2
        return {"select": kidx + qidx, "attn": kv + q_o}
    index = 2 * prob.d_idx * prob.h * int(lim.sum())
    attn = 4 * prob.d * prob.G * int(sel_tok.sum())
    return {"select": index, "attn": attn}


# ------------------------------------------------------------------- clocks
class ClockSampler:
    """Polls the GPU's SM clock and clock-event reasons through NVML every ~2 ms on a
    background thread; summary() keeps the samples taken inside the timed window."""

    # NVML clock-event reason bits (nvml.h)
    REASONS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
               "hw_thermal_slowdown": 0x40}

    def __init__(self, uuid: str | None):
        self.uuid = uuid
        self.samples = []
        self.window = None
        self.err = None
        self._stop = False
        self._thread = None

    def __enter__(self):
        import threading
        try:
            import pynvml
            pynvml.nvmlInit()
            h = (pynvml.nvmlDeviceGetHandleByUUID(self.uuid) if self.uuid
                 else pynvml.nvmlDeviceGetHandleByIndex(0))
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            reasons_fn = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
        except Exception as e:  # no NVML: report it, do not guess
            self.err = "nvml unavailable: %s" % e
            return self

        def poll():
            while not self._stop:
                try:
                    self.samples.append((time.perf_counter(),
                                         pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM),
                                         reasons_fn(h)))
                except Exception as e:
                    self.err = str(e)
                    return
                time.sleep(0.002)

        self._thread = threading.Thread(target=poll, daemon=True)
        self._thread.start()
        return self

    def mark(self, t0, t1):
        self.window = (t0, t1)

    def __exit__(self, *exc):
        self._stop = True
        if self._thread is not None:
            self._thread.join(timeout=2)

    def summary(self):
        if self.err and not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [self.err]}
        t0, t1 = self.window or (float("-inf"), float("inf"))
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        used = inside or self.samples[-3:]
        reasons = sorted({n for _, _, r in used for n, bit in self.REASONS.items() if r & bit})
        return {"sm_mhz": statistics.median(s[1] for s in used) if used else None,
                "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(inside),
                "source": "nvml, 2 ms polling, samples inside the timed region"}


# --------------------------------------------------------------- oracle arm
def oracle_sample(prob, x, budget_s: float, max_rows: int | None = None, collect=None):
    """Times the float64 oracle on a bounded sample: whole sequences for decode,
    query rows for prefill.  Returns (units processed, seconds, description); with
    ``collect`` (a list), appends (b, rows, ids, out) of every sampled sequence."""
    import numpy as np
    import oracle

    cfg1 = oracle.Config(1, prob.n_q, prob.max_kv, prob.H, prob.h, prob.d, prob.d_idx,
                         prob.block, prob.topk, causal=prob.causal, force_own=prob.force_own)
    units, secs, nseq, nrows = 0.0, 0.0, 0, 0
    rng = np.random.default_rng(0)
    for b in range(prob.batch):
        sl = x["seq_lens"][b:b + 1].cpu() if x["seq_lens"] is not None else None
        hb = {k: x[k][b:b + 1].cpu() for k in ("q", "k", "v", "q_idx", "k_idx")}
        if prob.is_decode:
            rows = [(0, 0)]
        else:
            n = max_rows or 64
            rows = [(0, int(t)) for t in sorted(rng.choice(prob.n_q, size=n, replace=False))]
        t0 = time.perf_counter()
        ids, _, _lse = oracle.forward(cfg1, hb["q"], hb["k"], hb["v"], hb["q_idx"], hb["k_idx"],
                                      seq_lens=sl, rows=rows)
        secs += time.perf_counter() - t0
        if collect is not None:
            collect.append((b, rows, ids, _))
        # work of the sampled rows, counted like the GPU's
        sub = prob.with_(batch=1)
        ids_t = torch.as_tensor(ids)
        if prob.is_decode:
            w = work_units(sub, {"seq_lens": sl}, ids_t.view(1, 1, prob.h, prob.topk))
            units += w["select"] + w["attn"]
        else:
            L, lim = positions(sub, sl, "cpu")
            tt = torch.as_tensor([r[1] for r in rows])
            lim_r = lim[0, tt]
            sel = selected_visible_tokens(sub, ids_t.view(1, len(rows), prob.h, prob.topk),
                                          lim_r.view(1, -1))
            units += 2 * prob.d_idx * prob.h * int(lim_r.sum()) + 4 * prob.d * prob.G * int(sel.sum())
        nseq += 1
        nrows += len(rows)
        if secs >= budget_s:
            break
    if prob.is_decode:
        desc = "%d of %d sequences (all %d groups, %d heads), full context" % (
            nseq, prob.batch, prob.h, prob.H)
    else:
        desc = "%d query rows (%d per sequence, %d sequences), all groups and heads" % (
            nrows, nrows // max(1, nseq), nseq)
    return units, secs, desc


def parity_stats(prob, x, ids, out, got, desc):
    """The GPU's ids and outputs of the last timed step against the oracle's on the
    CPU-baseline sample: rows whose ids are equal, rows that differ on a near tie
    (the oracle's k-th and (k+1)-th block scores within 1e-3 relative), and the
    output errors on rows with equal ids."""
    import numpy as np
    import oracle
    rows_n = same = near = 0
    errs = []
    ids_h = ids.cpu().numpy()
    out_h = out.float().cpu().numpy()
    for b, rows, oid, oout in got:
        tt = [t for _, t in rows]
        gi = ids_h[b, tt]                      # [nrows, h, topk]
        go = out_h[b, tt].reshape(oout.shape)  # [nrows, H, d]
        eq = (gi == oid).all(axis=-1)          # [nrows, h]
        rows_n += eq.size
        same += int(eq.sum())
        if not eq.all():
            sub = prob.with_(batch=1)
            cfg1 = oracle.Config(1, sub.n_q, sub.max_kv, sub.H, sub.h, sub.d, sub.d_idx,
                                 sub.block, sub.topk, causal=sub.causal, force_own=sub.force_own)
            sl = x["seq_lens"][b:b + 1].cpu() if x["seq_lens"] is not None else None
            sc = oracle.block_scores(cfg1, x["q_idx"][b:b + 1].cpu(), x["k_idx"][b:b + 1].cpu(),
                                     seq_lens=sl, rows=[(0, t) for t in tt])
            for i, g in zip(*np.nonzero(~eq)):
                v = np.sort(sc[i, g][np.isfinite(sc[i, g])])[::-1]
                k = min(prob.topk, len(v))
                if k < len(v) and (v[k - 1] - v[k]) / max(abs(v[k - 1]), abs(v[k]), 1e-6) < 1e-3:
                    near += 1
        for i in range(len(tt)):
            for g in range(prob.h):
                if eq[i, g]:
                    errs.append(np.abs(go[i, g * prob.G:(g + 1) * prob.G] -
                                       oout[i, g * prob.G:(g + 1) * prob.G]))
    e = np.concatenate([a.ravel() for a in errs]) if errs else np.zeros(1)
    return {"rows": rows_n, "ids_equal": same, "near_tie_rows": near,
            "other_mismatch_rows": rows_n - same - near, "max_abs": float(e.max()),
            "mean_abs": float(e.mean()), "tolerance": {"max_abs": 2e-2, "mean_abs": 2e-3},
            "oracle": "float64", "sample": desc}


def unit_of(prob):
    return ("GB/s", 1e9) if prob.is_decode else ("TFLOP/s", 1e12)


def run_reference(args, prob, world, rank):
    import oracle
    if rank != 0:
        return
    # The oracle samples whole sequences (decode) or query rows (prefill) of the
    # workload; drawing two sequences of it on the host is enough for that.
    sub = prob.with_(batch=min(prob.batch, 2))
    x = make_inputs(sub, device="cpu")
    prob = sub
    unit, scale = unit_of(prob)
    budget = 2.0
    for _ in range(args.warmup):
        oracle_sample(prob, x, 0.0, max_rows=8)
    units, secs = 0.0, 0.0
    desc = ""
    for _ in range(args.steps):
        u, s, desc = oracle_sample(prob, x, budget)
        units += u
        secs += s
    value = units / secs / scale
    cores = oracle.num_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": unit, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1), bf16 inputs widened to f64)",
        "config": {"workload": prob.name, **workload_config(prob)},
        "cpu_baseline": {"value": value, "unit": unit, "cores": cores, "kind": "oracle",
                         "sample": "each step: " + desc},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_config(prob):
    c = {"batch": prob.batch, "n_q": prob.n_q, "context": prob.max_kv, "H": prob.H, "h": prob.h,
         "d": prob.d, "d_idx": prob.d_idx, "block": prob.block, "topk": prob.topk,
         "causal": prob.causal, "force_own_block": prob.force_own}
    if prob.len_range:
        c["seq_len_range"] = list(prob.len_range)
    if prob.plant_frac:
        c["planted_block_frac"] = prob.plant_frac
    return c


# ----------------------------------------------------------------- our arm
def page_cache(prob, x, seed):
    """Moves k, v and k_idx into page pools of one block per page, the pages of all
    sequences shuffled over the pool, and adds the block table [batch, nblk]."""
    B = prob.block
    nb = (prob.max_kv + B - 1) // B
    g = torch.Generator(device="cpu").manual_seed(seed)
    table = torch.randperm(prob.batch * nb, generator=g).to(torch.int32).view(prob.batch, nb)
    table = table.to(x["k"].device)
    flat = table.view(-1).long()
    for name in ("k", "v", "k_idx"):
        t = x[name]
        tail = tuple(t.shape[2:])
        pool = torch.zeros((prob.batch * nb, B) + tail, dtype=t.dtype, device=t.device)
        for b in range(prob.batch):  # one sequence at a time bounds the extra memory
            blocks = torch.zeros((nb * B,) + tail, dtype=t.dtype, device=t.device)
            blocks[:t.shape[1]] = t[b]
            pool[flat[b * nb:(b + 1) * nb]] = blocks.view((nb, B) + tail)
            del blocks
        x[name] = pool
        del t
    x["block_table"] = table
    return x


def cache_row(prob, x, name, b, j):
    """The cache row of token j of sequence b (contiguous or paged)."""
    if "block_table" not in x:
        return x[name][b, j]
    page = int(x["block_table"][b, j // prob.block])
    return x[name][page, j % prob.block]


def run_ours(args, prob, world, rank, local):
    from block_sparse_gqa_03_b200 import msa

    dev = torch.device("cuda", local if world > 1 else 0)
    x = make_inputs(prob, device=dev, seed=prob.seed + rank)
    sl = x["seq_lens"]
    kw = dict(block=prob.block, causal=prob.causal, seq_lens=sl)
    if args.paged:
        x = page_cache(prob, x, seed=prob.seed + 7919 + rank)
        torch.cuda.empty_cache()
        kw.update(block_table=x["block_table"], max_kv=prob.max_kv)
    ids = torch.empty((prob.batch, prob.n_q, prob.h, prob.topk), dtype=torch.int32, device=dev)
    out = torch.empty_like(x["q"])
    ws = msa.Workspace(dev)
    stream = torch.cuda.current_stream(dev)

    # One step is one fused call (both stages, the kernels chained as programmatic
    # dependents); the per-stage times are measured in a separate pass.  With
    # --fused-select (prefill) the step is msa_index_topk (the top-k kept in the
    # index GEMM's epilogue) followed by msa_sparse_attn.
    if args.fused_select and prob.is_decode:
        raise SystemExit("--fused-select is a prefill option")

    def step():
        if args.fused_select:
            msa.msa_index_topk(x["q_idx"], x["k_idx"], topk=prob.topk,
                               force_own_block=prob.force_own, block_ids=ids, workspace=ws,
                               **kw)
            msa.msa_sparse_attn(x["q"], x["k"], x["v"], ids, out=out, workspace=ws, **kw)
        else:
            msa.msa_forward(x["q"], x["k"], x["v"], x["q_idx"], x["k_idx"], topk=prob.topk,
                            force_own_block=prob.force_own, out=out, block_ids=ids,
                            workspace=ws, **kw)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    assert msa.msa_get_device_status(ws) == msa.MSA_OK
    units = work_units(prob, x, ids)
    touched = units["select"] + units["attn"] if prob.is_decode else None

    K = args.steps
    props = torch.cuda.get_device_properties(dev)
    uuid = str(getattr(props, "uuid", "")) or None
    if uuid and not uuid.startswith("GPU-"):
        uuid = "GPU-" + uuid
    flush_buf = (torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
                 if args.l2_flush else None)

    def timed_loop():
        """K steps bracketed by a barrier and a synchronize on both sides; returns the
        per-step device times (ms) of the loop: one figure (loop / K) when the steps
        run back to back, K figures when the L2 is flushed before every step."""
        barrier(world)
        torch.cuda.synchronize(dev)
        if flush_buf is None:
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(K):
                step()
            e1.record(stream)
            torch.cuda.synchronize(dev)
            times = [e0.elapsed_time(e1) / K]
        else:
            ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(K)]
            for e0, e1 in ev:
                flush_buf.fill_(1.0)  # a write larger than L2, outside the timed span
                e0.record(stream)
                step()
                e1.record(stream)
            torch.cuda.synchronize(dev)
            times = [e0.elapsed_time(e1) for e0, e1 in ev]
        barrier(world)
        return times

    # the K-step loop is repeated until at least --min-ms of device time is timed,
    # so that the clock samples fall inside it and the spread is measured
    # (every rank must run the same number of loops: the largest calibration rules)
    calib = max_over_ranks(sum(timed_loop()) * (K if flush_buf is None else 1), world)
    repeats = max(1, min(args.max_repeats, -(-int(args.min_ms) // max(1, int(calib)))))
    step_times = []
    with ClockSampler(uuid) as clk:
        h0 = time.perf_counter()
        for _ in range(repeats):
            step_times.extend(timed_loop())
        clk.mark(h0, time.perf_counter())
    step_times.sort()

    def pct(q):
        return step_times[min(len(step_times) - 1, int(q * (len(step_times) - 1) + 0.5))]

    med_ms = max_over_ranks(statistics.median(step_times), world)
    step_stats = {"median_ms": med_ms, "p10_ms": max_over_ranks(pct(0.1), world),
                  "p90_ms": max_over_ranks(pct(0.9), world),
                  "mean_ms": max_over_ranks(statistics.mean(step_times), world),
                  "repeats": repeats, "steps_per_repeat": K,
                  "timed_ms": max_over_ranks(sum(step_times) * (K if flush_buf is None else 1),
                                             world),
                  "per": "K-step loop / K" if flush_buf is None else "step"}

    # per-kernel times (for the roofline of the dominant kernel), measured apart
    # from the timed region with events around each call: the index scan alone
    # (msa_block_scores), scan + top-k (msa_index_select) and the attention call
    # (msa_sparse_attn: its merge-counter memset and kernel; prefill: the whole
    # KV-major stage)
    scores_buf = torch.empty((prob.batch, prob.n_q, prob.h, prob.nblk), dtype=torch.float32,
                             device=dev)
    ks = max(5, min(20, int(200.0 / max(med_ms, 1e-3))))
    calls = {
        "scan": lambda: msa.msa_block_scores(x["q_idx"], x["k_idx"], block=prob.block,
                                             causal=prob.causal, seq_lens=sl,
                                             block_scores=scores_buf, workspace=ws,
                                             **{k: kw[k] for k in ("block_table", "max_kv")
                                                if k in kw}),
        "select": lambda: msa.msa_index_select(x["q_idx"], x["k_idx"], topk=prob.topk,
                                               force_own_block=prob.force_own, block_ids=ids,
                                               workspace=ws, **kw),
        "attn": lambda: msa.msa_sparse_attn(x["q"], x["k"], x["v"], ids, out=out, workspace=ws,
                                            **kw),
    }
    stage = {}
    for name, fn in calls.items():
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(ks)]
        fn()
        for e0, e1 in ev:
            if flush_buf is not None:
                flush_buf.fill_(1.0)
            e0.record(stream)
            fn()
            e1.record(stream)
        torch.cuda.synchronize(dev)
        stage[name] = statistics.median(e0.elapsed_time(e1) for e0, e1 in ev)
    assert msa.msa_get_device_status(ws) == msa.MSA_OK
    sel_ms, attn_ms = stage["select"], stage["attn"]
    # the top-k time as select - scan holds for decode only: the scan-only call
    # writes every block's score (-inf past the frontier), which for a causal
    # prefill is about twice what the scan inside select writes
    kern_ms = {"scan": stage["scan"],
               "topk": max(0.0, stage["select"] - stage["scan"]) if prob.is_decode else None,
               "attn": stage["attn"]}
    ms_per_step = med_ms
    unit, scale = unit_of(prob)
    total_units = (units["select"] + units["attn"]) * world
    value = total_units / (ms_per_step * 1e-3) / scale

    # End to end through the public API: inputs from pinned host memory, the
    # result read back, every step.
    e2e = None if args.no_e2e else run_e2e(args, prob, x, dev, world, msa, kw)

    p_sel = msa.make_params(batch=prob.batch, n_q=prob.n_q, max_kv=prob.max_kv, H=prob.H,
                            h=prob.h, d=prob.d, d_idx=prob.d_idx, block=prob.block,
                            topk=prob.topk, causal=prob.causal, q=x["q"], k=x["k"], v=x["v"],
                            q_idx=x["q_idx"], k_idx=x["k_idx"], out=out)
    launches_per_step = (msa.msa_launch_count(p_sel, msa.MSA_OP_INDEX_TOPK) +
                         msa.msa_launch_count(p_sel, msa.MSA_OP_SPARSE_ATTN)
                         if args.fused_select else
                         msa.msa_launch_count(p_sel, msa.MSA_OP_FORWARD))

    peaks, peak_kind = load_peaks()
    if prob.is_decode:
        names = {"scan": "index_scan_stream_kernel", "attn": "sparse_attn_stream_kernel"}
        work = {"scan": units["select"], "attn": units["attn"]}
    else:
        names = {"scan": "index_score_tc_kernel",
                 "attn": "sparse attention stage (inverted index, kv_attn_kernel, combine)"}
        work = {"scan": units["select"], "attn": units["attn"]}
    dom = "attn" if kern_ms["attn"] >= kern_ms["scan"] else "scan"

    def roof_of(k):
        if prob.is_decode:
            r = {"bound": "hbm", "achieved": work[k] / (kern_ms[k] * 1e-3) / 1e9,
                 "peak": peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]), "unit": "GB/s"}
        else:
            r = {"bound": "tensor", "achieved": work[k] / (kern_ms[k] * 1e-3) / 1e12,
                 "peak": peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]),
                 "unit": "TFLOP/s"}
            sus = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
            r["frac_of_sustained_peak"] = r["achieved"] / sus
        r["frac"] = r["achieved"] / r["peak"]
        r["kernel"] = names[k]
        r["ms"] = kern_ms[k]
        return r

    # the captured traffic holds for the workload as defined (not for overridden sizes)
    stock = prob == WORKLOADS.get(prob.name) and not args.paged
    roof = roof_of(dom)
    roof["traffic"] = TRAFFIC.get((prob.name, dom)) if stock else None
    roof["peak_source"] = "of %s (%s)" % (peak_kind, "copy" if prob.is_decode else "burst bf16")
    other = "scan" if dom == "attn" else "attn"
    o = roof_of(other)
    o["traffic"] = TRAFFIC.get((prob.name, other)) if stock else None
    roof["other_kernels"] = [o, {"kernel": "topk_%s_kernel" % ("cta" if prob.nblk > 1024
                                                               else "warp"),
                                 "ms": kern_ms["topk"]}]
    if not prob.is_decode:
        # the whole step against the dense bf16 peak (the prefill target)
        roof["step_frac_of_peak"] = value / roof["peak"]

    line = {
        "metric": METRIC, "value": value, "unit": unit, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16%s)" % (", planted blocks" if prob.plant_frac else ""),
        "config": {"workload": prob.name, **workload_config(prob),
                   "kv_cache": "paged (one block per page, shuffled pool)" if args.paged
                   else "contiguous",
                   "l2": ("flushed before every step (%d MiB written), each step timed alone"
                          % (L2_FLUSH_BYTES >> 20) if args.l2_flush else
                          "no flush: inputs larger than L2 (%.2f GB touched per step)"
                          % (touched / 1e9) if touched else
                          "no flush: inputs larger than L2"),
                   "parallelism": "replicas" if world > 1 else "single GPU",
                   "select": "msa_index_topk (streaming top-k)" if args.fused_select
                   else "index GEMM/scan + top-k kernel"},
        "us_per_step": 1e3 * ms_per_step,
        "step_ms": step_stats,
        "stage_ms": {"index_scan": stage["scan"], "index_select": sel_ms, "sparse_attn": attn_ms},
        "roofline": roof,
        "e2e": e2e,
        "gpu_launches": launches_per_step * K * repeats,
    }
    if prob.is_decode:
        line["tokens_per_s"] = prob.batch * world / (ms_per_step * 1e-3)
    if rank == 0:
        line["clocks"] = clk.summary()
        if world == 1 and not args.no_cpu_baseline and not args.paged:
            import oracle
            got = []
            u, s, desc = oracle_sample(prob, {k: v for k, v in x.items()}, args.cpu_budget,
                                       collect=got)
            line["cpu_baseline"] = {"value": u / s / scale, "unit": unit,
                                    "cores": oracle.num_threads(), "kind": "oracle",
                                    "sample": desc}
            line["parity"] = parity_stats(prob, x, ids, out, got, desc)
        print(json.dumps(line), flush=True)


def run_e2e(args, prob, x, dev, world, msa, kw):
    """Same metric through the public API with host buffers: pinned host -> device
    copies of the step's inputs, the calls, and the output read back, inside the
    timed region (decode: the step replayed as a captured CUDA graph unless
    --e2e-eager)."""
    stream = torch.cuda.current_stream(dev)
    out_dev = torch.empty_like(x["q"])
    out_host = torch.empty(out_dev.shape, dtype=out_dev.dtype, pin_memory=True)
    d2h = out_host.numel() * out_host.element_size()
    ws = msa.Workspace(dev)
    nsteps = max(1, min(args.steps, 20))
    if prob.is_decode:
        # A decode step's inputs are the new token's queries and its K/V/K_idx rows:
        # packed in one pinned buffer, copied once, the rows written into the
        # resident cache at position L_b - 1 by msa_append_kv, then msa_forward.
        # (The rows are the cache's own, so the cache is unchanged step to step.)
        # Copying the attention queries on a second stream beside msa_index_select,
        # then msa_sparse_attn, measured slower (218 against 210 us at 128K): the
        # extra dependency and the merge-counter memset cost more than the copy.
        L = (x["seq_lens"].cpu().tolist() if x["seq_lens"] is not None
             else [prob.max_kv] * prob.batch)
        parts = {"q": x["q"], "q_idx": x["q_idx"]}
        for n in ("k", "v", "k_idx"):
            parts[n + "_new"] = torch.stack([cache_row(prob, x, n, b, L[b] - 1)
                                             for b in range(prob.batch)]).unsqueeze(1)
        flat = [t.reshape(-1) for t in parts.values()]
        host = torch.cat(flat).cpu().pin_memory()
        staging = torch.empty_like(host, device=dev)
        views, off = {}, 0
        for n, t in parts.items():
            views[n] = staging[off:off + t.numel()].view(t.shape)
            off += t.numel()
        h2d = host.numel() * host.element_size()
        akw = {k: kw[k] for k in ("block", "seq_lens", "block_table", "max_kv") if k in kw}

        def one():
            staging.copy_(host, non_blocking=True)
            msa.msa_append_kv(x["k"], x["v"], x["k_idx"], views["k_new"], views["v_new"],
                              views["k_idx_new"], workspace=ws, **akw)
            msa.msa_forward(views["q"], x["k"], x["v"], views["q_idx"], x["k_idx"],
                            topk=prob.topk, force_own_block=prob.force_own, out=out_dev,
                            workspace=ws, **kw)
            out_host.copy_(out_dev, non_blocking=True)
    elif x["seq_lens"] is None and "block_table" not in kw:
        # Prefill as a chunked prefill through the same API: the inputs are copied
        # chunk by chunk in token order on a copy stream, msa_forward runs query
        # chunk c (the context up to the chunk's last query) as soon as its rows
        # have landed, and each chunk's output is read back on a third stream, so
        # that the copies overlap the compute.
        names = ["q", "k", "v", "q_idx", "k_idx"]
        host = {n: x[n].cpu().pin_memory() for n in names}
        h2d = sum(t.numel() * t.element_size() for t in host.values())
        qc = min(prob.n_q, 16384 if prob.batch == 1 else 8192)
        off = prob.max_kv - prob.n_q  # query t sits at position off + t
        chunks = []
        for c0 in range(0, prob.n_q, qc):
            c1 = min(c0 + qc, prob.n_q)
            k0 = 0 if c0 == 0 else off + c0
            chunks.append((c0, c1, k0, off + c1,
                           torch.full((prob.batch,), off + c1, dtype=torch.int32, device=dev)))
        s_copy, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        landed = [torch.cuda.Event() for _ in chunks]
        done = [torch.cuda.Event() for _ in chunks]
        ckw = {k: v for k, v in kw.items() if k != "seq_lens"}

        def one():
            s_copy.wait_stream(stream)
            with torch.cuda.stream(s_copy):
                for (c0, c1, k0, k1, _), ev in zip(chunks, landed):
                    for b in range(prob.batch):
                        for n in ("q", "q_idx"):
                            x[n][b, c0:c1].copy_(host[n][b, c0:c1], non_blocking=True)
                        for n in ("k", "v", "k_idx"):
                            x[n][b, k0:k1].copy_(host[n][b, k0:k1], non_blocking=True)
                    ev.record(s_copy)
            for (c0, c1, _, _, sl), ev, dn in zip(chunks, landed, done):
                stream.wait_event(ev)
                msa.msa_forward(x["q"][:, c0:c1], x["k"], x["v"], x["q_idx"][:, c0:c1], x["k_idx"],
                                topk=prob.topk, force_own_block=prob.force_own,
                                out=out_dev[:, c0:c1], workspace=ws, seq_lens=sl, **ckw)
                dn.record(stream)
                s_out.wait_event(dn)
                with torch.cuda.stream(s_out):
                    for b in range(prob.batch):
                        out_host[b, c0:c1].copy_(out_dev[b, c0:c1], non_blocking=True)
            stream.wait_stream(s_out)
    else:
        names = ["q", "k", "v", "q_idx", "k_idx"]
        host = {n: x[n].cpu().pin_memory() for n in names}
        h2d = sum(t.numel() * t.element_size() for t in host.values())

        def one():
            for n in names:
                x[n].copy_(host[n], non_blocking=True)
            msa.msa_forward(x["q"], x["k"], x["v"], x["q_idx"], x["k_idx"], topk=prob.topk,
                            force_own_block=prob.force_own, out=out_dev, workspace=ws, **kw)
            out_host.copy_(out_dev, non_blocking=True)

    one()
    torch.cuda.synchronize(dev)
    step, graphed = one, False
    if prob.is_decode and not args.e2e_eager:
        # A decode step as a serving loop runs it: captured once as a CUDA graph (the
        # pinned-memory copies, msa_append_kv and msa_forward's kernels with their
        # programmatic dependencies) and replayed every step; the copies stay inside.
        graph = torch.cuda.CUDAGraph()
        # thread-local capture: other threads (a process group's watchdog, the clock
        # sampler) may use CUDA meanwhile
        with torch.cuda.graph(graph, capture_error_mode="thread_local"):
            one()
        step, graphed = graph.replay, True
        nsteps = max(1, min(args.steps, 400))
        step()
        torch.cuda.synchronize(dev)
    barrier(world)
    s0 = torch.cuda.Event(enable_timing=True)
    s1 = torch.cuda.Event(enable_timing=True)
    s0.record(stream)
    for _ in range(nsteps):
        step()
    s1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    ms = max_over_ranks(s0.elapsed_time(s1), world) / nsteps
    ids = torch.empty((prob.batch, prob.n_q, prob.h, prob.topk), dtype=torch.int32, device=dev)
    msa.msa_index_select(x["q_idx"], x["k_idx"], topk=prob.topk, force_own_block=prob.force_own,
                         block_ids=ids, workspace=ws, **kw)
    u = work_units(prob, x, ids)
    unit, scale = unit_of(prob)
    return {"value": (u["select"] + u["attn"]) * world / (ms * 1e-3) / scale, "unit": unit,
            "ms_per_step": ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "steps": nsteps, "cuda_graph": graphed}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default=DEFAULT_WORKLOAD)
    ap.add_argument("--cpu-budget", type=float, default=10.0)
    ap.add_argument("--min-ms", type=float, default=200.0,
                    help="repeat the K-step loop until this much device time is timed")
    ap.add_argument("--max-repeats", type=int, default=400)
    ap.add_argument("--fused-select", action="store_true",
                    help="prefill: select with msa_index_topk (top-k in the index GEMM's "
                         "epilogue) instead of the GEMM + top-k kernels")
    ap.add_argument("--l2-flush", action="store_true",
                    help="write a buffer larger than L2 before every step and time each step "
                         "alone")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-eager", action="store_true",
                    help="decode e2e: issue the step's calls one by one instead of replaying "
                         "them as a captured CUDA graph")
    ap.add_argument("--batch", type=int, default=0,
                    help="override the workload's batch (for small profiling captures)")
    ap.add_argument("--seq", type=int, default=0,
                    help="override the sequence length (prefill: queries and context; decode: "
                         "context) for small profiling captures")
    ap.add_argument("--paged", action="store_true",
                    help="keep K, V and K_idx in a paged cache (one block per page, pages "
                         "shuffled over the pool) addressed through a block table")
    ap.add_argument("--queries", type=int, default=0,
                    help="prefill only: keep the context and take the last N positions as the "
                         "query rows (chunked prefill), for small profiling captures")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    prob = WORKLOADS[args.workload]
    if args.batch:
        prob = prob.with_(batch=args.batch)
    if args.seq:
        if prob.is_decode:
            lr = prob.len_range
            prob = prob.with_(max_kv=args.seq,
                              len_range=None if lr is None else (min(lr[0], args.seq), args.seq))
        else:
            prob = prob.with_(n_q=args.seq, max_kv=args.seq)
    if args.queries and not prob.is_decode:
        prob = prob.with_(n_q=min(args.queries, prob.max_kv))
    world, rank, local = dist_setup(args)
    try:
        if args.impl == "reference":
            run_reference(args, prob, world, rank)
        else:
            run_ours(args, prob, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
