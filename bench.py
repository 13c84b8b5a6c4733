"""Benchmark of the WorldAttention per-layer HKV + HSA step on B200.

One step = page-level retrieval (hkv_select_pages) + active-cache gather
(hkv_gather, with the fused 128-row K pooling) + hsa_forward (pooling, block
selection, Linformer projection and attention, sparse attention with the gated
merge).  The default workload is the largest one: the 14B-shaped 720p step (40
heads, d = 128, a 10800-query chunk, 12 history pages of 28800 tokens resident in
HBM, Kp = 4, r = 512).  ``--workload I`` selects another (0 tiny, 1 Wan-1.3B
480p, 2 14B 480p, 3 14B 720p, 4 90-second horizon with host-pinned pages).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--workload I]

Prints one JSON line (rank 0).  N > 1 runs one independent replica per GPU
(torchrun, NCCL for the barrier and the max-over-ranks timing only).
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "HSA layer query-tokens/s + eff. TFLOP/s on 1 B200; % tensor/HBM roofline"
UNIT = "query-tokens/s"
DEFAULT_WORKLOAD = 3

TRAFFIC = {
    # dram__bytes_read.sum + dram__bytes_write.sum of one launch, from an ncu capture at
    # TRAFFIC_WORKLOAD (the summaries under profiles/), with the rows x heads x d of KV
    # that launch streamed; valid while the kernel's source section is unchanged (sha).
    # Another workload scales the bytes by its own launch's rows x heads x d.
    "attention_merge": {"file": "attn_tc.cu", "section": "kernel", "sha": "2da5f949c952ab3f",
                        "bytes": 277418240 + 18491136, "rows": "cached"},
}
TRAFFIC_WORKLOAD = 1  # synth.SHAPES index of the captured workload (Wan-1.3B 480p)


def launch_rows(name, shape):
    """KV rows one launch of kernel `name` streams."""
    return shape.Lc


def traffic_of(name, shape):
    """Per-launch DRAM traffic of kernel `name` at `shape`, or None (no capture, or the
    kernel's source changed since the capture)."""
    tr = TRAFFIC.get(name)
    if not tr or tr["sha"] != section_sha(os.path.join(ROOT, "hybrid_sparse_attention_hkv_b200", "csrc", tr["file"]),
                                          tr["section"]):
        return None
    import synth
    ref = synth.SHAPES[TRAFFIC_WORKLOAD]
    f = (launch_rows(name, shape) * shape.H * shape.d) / (launch_rows(name, ref) * ref.H * ref.d)
    return int(round(tr["bytes"] * f))


SECTION_MARK = "// ------------------------------------------------------------------ "


def section_sha(path, section):
    """sha256 prefix of the text from the `section` marker line to the next marker (or the end)."""
    with open(path) as f:
        text = f.read()
    start = text.find(SECTION_MARK + section)
    if start < 0:
        return None
    nxt = text.find(SECTION_MARK, start + len(SECTION_MARK))
    return hashlib.sha256(text[start:nxt if nxt >= 0 else len(text)].encode()).hexdigest()[:16]


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            m = json.load(f)
        return {"hbm_gbs": m["hbm_gbs"], "bf16_tflops": m["bf16_tflops"],
                "bf16_tflops_sustained": m.get("bf16_tflops_sustained", m["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ------------------------------------------------------------------ work model
def step_work(shape):
    """Algorithmic FLOPs and bytes of one step's dense parts (the sparse branch is
    counted from the selection by exact_pairs)."""
    H, d, Lq, Lc, r = shape.H, shape.d, shape.Lq, shape.Lc, shape.r
    L = Lc + Lq
    return {
        "proj_flops": H * 4.0 * r * L * d,             # EK and FV: 2 * (2 r L d) per head
        "proj_chunk_flops": H * 4.0 * r * Lq * d,      # the chunk's own rows only (history prepared)
        "proj_hist_flops": H * 4.0 * r * Lc * d,       # the cached rows only
        "lin_attn_flops": H * 4.0 * Lq * r * d,        # Q EK^T and P FV
        "gather_bytes": 4.0 * Lc * H * d * 2,          # read + write of K and V pages
        "proj_bytes": 2.0 * L * H * d * 2 + 2.0 * r * L * 2,
        "pool_bytes": 2.0 * Lq * H * d * 2,            # Q and Kq read once
        "select_pages_bytes": Lq * H * d * 2.0,        # Q read once
    }


def kernels_in_scope(name, shape, joint=False):
    """Kernels one traced library call launches inside a step.  The block selection
    runs its scores kernel once per map (the inter map only when there is a cached
    KV; one map in joint mode) and then its ranking kernel; the page store's fetch
    updates the residency on the device and then launches its copy kernel.  Every
    other call of the step launches one kernel."""
    if name == "block_select":
        maps = 1 if joint else (1 if shape.Lc > 0 else 0) + 1
        return maps + 1
    if name == "store_fetch":
        return 2
    return 1


def exact_pairs(shape, sel_bufs):
    """Selected query-key pairs counted from the selection lists (partial blocks exact)."""
    import numpy as np
    H, Lq, Lc = shape.H, shape.Lq, shape.Lc
    ic = sel_bufs.inter_cnt.cpu().numpy()
    ii = sel_bufs.inter_idx.cpu().numpy()
    qc = sel_bufs.intra_cnt.cpu().numpy()
    qi = sel_bufs.intra_idx.cpu().numpy()
    kc_size = np.array([min(128, Lc - 128 * j) for j in range(-(-Lc // 128))], dtype=np.float64)
    kq_size = np.array([min(64, Lq - 64 * j) for j in range(-(-Lq // 64))], dtype=np.float64)
    pairs = 0.0
    for h in range(H):
        for i in range(ic.shape[1]):
            pairs += min(128, Lq - 128 * i) * kc_size[ii[h, i, :ic[h, i]]].sum()
        for i in range(qc.shape[1]):
            pairs += min(64, Lq - 64 * i) * kq_size[qi[h, i, :qc[h, i]]].sum()
    return pairs, float(ic.sum()) / max(1, ic.size * len(kc_size)), float(qc.sum()) / max(1, qc.size * len(kq_size))


def kept_fraction_per_head(shape, sel_bufs):
    """Per head, the fraction of (query block, key block) pairs kept in the inter and
    in the intra map (the head-adaptive threshold keeps more blocks at larger tau_h)."""
    H, Lq, Lc = shape.H, shape.Lq, shape.Lc
    nkc, nkq = -(-Lc // 128), -(-Lq // 64)
    ic = sel_bufs.inter_cnt.cpu().double().reshape(H, -1)
    qc = sel_bufs.intra_cnt.cpu().double().reshape(H, -1)
    inter = (ic.sum(1) / max(1, ic.shape[1] * nkc)).tolist()
    intra = (qc.sum(1) / max(1, qc.shape[1] * nkq)).tolist()
    return [round(v, 4) for v in inter], [round(v, 4) for v in intra]


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi clock / throttle-reason samples; mark() brackets the timed region."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index=0):
        self.index = index
        self.proc = None
        self.lines = []
        self.err = ""
        self.marks = []

    def start(self, wait_s=5.0):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True)
        except OSError as e:
            self.err = str(e)
            self.proc = None
            return
        self.t = threading.Thread(target=self._read, daemon=True)
        self.t.start()
        t0 = time.time()
        while not self.lines and time.time() - t0 < wait_s and self.proc.poll() is None:
            time.sleep(0.02)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def mark(self):
        self.marks.append(len(self.lines))

    def stop(self):
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [f"nvidia-smi unavailable: {self.err}"]}
        self.proc.terminate()
        try:
            _, err = self.proc.communicate(timeout=5)
            self.err = (err or "").strip()[:200]
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.t.join(timeout=2)
        lo, hi = (self.marks + [0, len(self.lines)])[:2] if len(self.marks) >= 2 else (0, len(self.lines))
        window = self.lines[lo:max(hi, lo + 1)] or self.lines[-1:]
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in window:
            f = [x.strip() for x in ln.split(",")]
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
        out = {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
               "samples": len(sm)}
        if not sm and self.err:
            out["error"] = self.err
        return out


# ------------------------------------------------------------------ CPU oracle timing
def oracle_summaries(x, shape):
    """Page summaries (computed when a page is sealed, outside the step)."""
    import numpy as np
    import oracle
    return np.stack([oracle.page_summary(x.pages_k[p], np.float32) for p in range(shape.NP)])


def oracle_sample_plan(shape, small=False):
    """The bounded sample the fp64 oracle is timed on: (heads, query rows).  Whole step
    for the tiny workload; otherwise the first, middle and last head (tau 1.00, ~0.68,
    0.35) on the rows of three 128-row query blocks (first, middle, last); `small`
    (one step of the reference arm) takes one head and one query block."""
    import numpy as np
    if shape.Lq <= 512 and shape.H <= 4:
        return list(range(shape.H)), None
    nQ = -(-shape.Lq // 128)
    if small:
        return [0], np.arange(0, min(128, shape.Lq))
    heads = sorted({0, shape.H // 2, shape.H - 1})
    blocks = sorted({0, nQ // 2, nQ - 1})
    rows = np.concatenate([np.arange(128 * b, min(128 * (b + 1), shape.Lq)) for b in blocks])
    return heads, rows


def oracle_step_sample(x, shape, kbar, heads, rows):
    """Time the fp64 oracle, phase by phase, on a bounded sample of one step:
      t_r            page retrieval + gather (whole, all heads);
      t_fixed[h]     block selection (whole maps) + Linformer projection (whole) of head h;
      t_rows[h]      both attention branches and the merge of head h on `rows`.
    Step time (extrapolated unless the sample is the whole step):
      t_r + (H / len(heads)) * sum_h (t_fixed[h] + t_rows[h] * Lq / len(rows))."""
    import numpy as np
    import oracle
    nrows = shape.Lq if rows is None else len(rows)
    t0 = time.perf_counter()
    sel, _ = oracle.select_pages(kbar, x.Q, shape.Kp)
    Kc = oracle.gather_pages(x.pages_k, sel)
    Vc = oracle.gather_pages(x.pages_v, sel)
    t_r = time.perf_counter() - t0
    per_head = 0.0
    timed = t_r
    for h in heads:
        hs = [h]
        Qh, Kch, Vch, Kqh, Vqh = x.Q[:, hs], Kc[:, hs], Vc[:, hs], x.Kq[:, hs], x.Vq[:, hs]
        t0 = time.perf_counter()
        selh = oracle.block_select(Qh, Kch, Kqh, x.tau[hs])
        EK, FV = oracle.linear_projection(x.E, x.F, Kch, Kqh, Vch, Vqh)
        t1 = time.perf_counter()
        o_s = oracle.sparse_attention(Qh, Kch, Vch, Kqh, Vqh, selh.inter, selh.intra, rows=rows)
        o_l = oracle.linear_attention(Qh, EK, FV, rows=rows)
        oracle.gated_merge(o_s, o_l, x.z[hs])
        t2 = time.perf_counter()
        per_head += (t1 - t0) + (t2 - t1) * shape.Lq / nrows
        timed += t2 - t0
    t_step = t_r + per_head * shape.H / len(heads)
    whole = len(heads) == shape.H and nrows == shape.Lq
    if whole:
        sample = "the whole step: page retrieval, gather, block selection, both branches and merge, all heads and rows"
    else:
        sample = (f"page retrieval + gather (whole); heads {list(heads)}: block selection and projection (whole), "
                  f"both branches + merge on {nrows} of {shape.Lq} query rows; step time extrapolated as "
                  f"t_retrieval + (H/heads) * sum_h (t_select_proj + t_rows * Lq/rows)")
    return {"t_step": t_step, "sample": sample, "timed_seconds": timed, "extrapolated": not whole}


def blas_threads():
    try:
        import threadpoolctl
        return max([i.get("num_threads", 1) for i in threadpoolctl.threadpool_info()] + [1])
    except Exception:  # noqa: BLE001
        return os.cpu_count() or 1


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def _time_ms(fn, n, stream=None):
    """Mean device time (ms) of n calls of fn on the current stream (CUDA events)."""
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(s)
    for _ in range(n):
        fn()
    e1.record(s)
    e1.synchronize()
    return e0.elapsed_time(e1) / n


def host_tier_report(ds, shape, args, host_gbs):
    """The host-pinned history three ways: the step as timed (pages fetched into the
    store's HBM slots; after the warm-up the selected pages are resident, as when
    consecutive chunks retrieve the same pages), the gather straight from the host
    tier (zero-copy), and a cold fetch (every selected page promoted over the link)."""
    import hybrid_sparse_attention_hkv_b200 as hsa
    st, store = ds.step, ds.store
    n = max(3, min(args.steps, 10))
    kp, vp = ds.host_tables
    zero_copy = _time_ms(lambda: hsa.hkv_gather(kp, vp, st.sel, shape.Kp, shape.P_tok, shape.H, shape.d, st.Kc, st.Vc,
                                                st.ws, st.kbar128), n)

    def cold():
        hsa.load_library().hkv_store_init(ctypes.byref(store.desc), None)
        store.fetch(st.sel, st.ws)

    cold_ms = _time_ms(cold, n)
    store_gather = _time_ms(lambda: hsa.hkv_gather(st.page_k_ptrs, st.page_v_ptrs, st.sel, shape.Kp, shape.P_tok,
                                                   shape.H, shape.d, st.Kc, st.Vc, st.ws, st.kbar128), n)
    store.fetch(st.sel, st.ws)  # resident again for what follows
    page_bytes = 2.0 * shape.P_tok * shape.H * shape.d * 2  # K and V of one page
    return {"slots": store.S, "pages": shape.NP,
            "zero_copy_gather_ms": zero_copy, "zero_copy_GBps": shape.Kp * page_bytes / (zero_copy / 1e3) / 1e9,
            "cold_fetch_ms": cold_ms, "cold_fetch_GBps": shape.Kp * page_bytes / (cold_ms / 1e3) / 1e9,
            "resident_gather_ms": store_gather, "host_link_copy_GBps": host_gbs,
            "note": "value / ms_per_step: steady state with the selected pages resident in the HBM slots"}


def reuse_report(ds, shape, args):
    """Multi-step reuse: retrieval, gather and the history's projection once per chunk
    (prepare_chunk), then one hsa_forward_reuse per denoising step."""
    st = ds.step
    n = max(3, min(args.steps, 20))
    chunk_ms = _time_ms(lambda: st.prepare_chunk(ds.Q, ds.E, ds.F, ds.e_cur, ds.e_seg, ds.seg_begin), n)
    step_ms = _time_ms(lambda: st.denoise_step(ds.Q, ds.Kq, ds.Vq, ds.tau, ds.z, ds.E, ds.F), n)
    return {"chunk_ms": chunk_ms, "denoise_step_ms": step_ms,
            "query_tokens_per_s_4_steps": 4 * shape.Lq / ((chunk_ms + 4 * step_ms) / 1e3),
            "note": "chunk = page retrieval + gather + the cached KV's Linformer products; step = block selection, "
                    "the chunk's projection, both branches and the merge; L2 not flushed"}


def measure_host_link(dev, nbytes=256 << 20, reps=5):
    """Best pinned host -> device copy bandwidth (GB/s) over `reps` copies of `nbytes`."""
    import torch
    src = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
    dst = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    best = 0.0
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        dst.copy_(src, non_blocking=True)
        e1.record()
        e1.synchronize()
        best = max(best, nbytes / (e0.elapsed_time(e1) / 1e3) / 1e9)
    del src, dst
    return best


# ------------------------------------------------------------------ distributed plumbing
def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        backend = os.environ.get("HSA_BENCH_BACKEND", "nccl")
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(value, world, device="cpu"):
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ arms
def run_reference(args, shape, rank, world):
    """The oracle as it stands, on the host cores: every step times a bounded sample
    of the step (one head, one query block, plus the whole page retrieval and
    gather) and extrapolates the step time from it; the line says so."""
    if rank != 0:
        return None
    import synth
    x = synth.make_inputs(shape, synth.seed_of(args.workload))
    kbar = oracle_summaries(x, shape)
    heads, rows = oracle_sample_plan(shape, small=True)
    for _ in range(args.warmup):
        oracle_step_sample(x, shape, kbar, heads, rows)
    ts, timed = [], 0.0
    r = None
    for k in range(args.steps):
        hk = [k % shape.H] if len(heads) < shape.H else heads  # rotate the sampled head
        r = oracle_step_sample(x, shape, kbar, hk, rows)
        ts.append(r["t_step"])
        timed += r["timed_seconds"]
    t_step = statistics.mean(ts)
    value = shape.Lq / t_step
    cores = blas_threads()
    sample = r["sample"] + "; the sampled head rotates over the steps"
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": t_step * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
        "config": workload_config(shape, args),
        "extrapolated": r["extrapolated"], "timed_seconds": timed,
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample,
                         "extrapolated": r["extrapolated"], "timed_seconds": timed, "cpu": cpu_model()},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def input_bytes(shape):
    """Bytes of one step's inputs: the page store, Q / Kq / Vq and E / F (bf16)."""
    hd = shape.H * shape.d
    return 2.0 * (2 * shape.NP * shape.P_tok * hd + 3 * shape.Lq * hd + 2 * shape.r * shape.L)


def workload_config(shape, args):
    return {"workload": shape.name, "H": shape.H, "d": shape.d, "Lq": shape.Lq, "Lc": shape.Lc, "L": shape.L,
            "P_tok": shape.P_tok, "NP": shape.NP, "Kp": shape.Kp, "r": shape.r, "block_inter": 128,
            "block_intra": 64, "tau": "1.00 -> 0.35 linear across heads", "pages": "host-pinned" if shape.host_pages else "HBM",
            "l2": f"flushed between timed steps (256 MiB write); inputs {input_bytes(shape) / 1e9:.2f} GB",
            "parallelism": f"replicas x{getattr(args, 'gpus', 1)}"}


def run_gpu(args, shape, rank, world, local):
    import numpy as np
    import torch

    import synth
    import hybrid_sparse_attention_hkv_b200 as hsa
    from synth.device import DeviceStep

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    seed = synth.seed_of(args.workload) + rank  # each replica its own seeded inputs
    # a history on the host tier is read through the tiered page store (Kp + 4 HBM slots)
    ds = DeviceStep(shape, seed, store_slots=(shape.Kp + 4) if shape.host_pages else 0)
    st = ds.step
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def one_step():
        ds.run()

    for _ in range(args.warmup):
        flush.zero_()
        one_step()
    torch.cuda.synchronize()

    trace = hsa.KernelTrace(max_kernels=64 * args.steps)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    clocks = ClockSampler(local)
    clocks.start()
    barrier(world)
    torch.cuda.synchronize()
    clocks.mark()
    with trace:
        for k in range(args.steps):
            flush.zero_()
            starts[k].record(stream)
            one_step()
            ends[k].record(stream)
    torch.cuda.synchronize()
    clocks.mark()
    clk = clocks.stop()
    barrier(world)
    t_steps = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    t_total = sum(t_steps) / 1e3
    t_max = max_over_ranks(t_total, world, dev if world > 1 and os.environ.get("HSA_BENCH_BACKEND", "nccl") == "nccl" else "cpu")
    per_kernel = {}
    launches = 0
    for name, ms in trace.results():
        launches += kernels_in_scope(name, shape)
        d = per_kernel.setdefault(name, {"launches": 0, "ms": 0.0})
        d["launches"] += 1
        d["ms"] += ms
    value = world * shape.Lq * args.steps / t_max
    ms_per_step = t_max / args.steps * 1e3

    # e2e: host buffers through the public API, copies inside the timed region.  As a
    # serving loop would, the host-to-device copy of step k + 1's inputs and the
    # device-to-host copy of step k - 1's output run on their own streams while step k
    # computes (double-buffered device inputs and outputs); the timed region runs from
    # the first input copy to the last output copy.
    hQ = ds.Q.cpu().pin_memory()
    hK = ds.Kq.cpu().pin_memory()
    hV = ds.Vq.cpu().pin_memory()
    hout = [torch.empty(st.out.shape, dtype=st.out.dtype).pin_memory() for _ in range(2)]
    dQ = [ds.Q, torch.empty_like(ds.Q)]
    dK = [ds.Kq, torch.empty_like(ds.Kq)]
    dV = [ds.Vq, torch.empty_like(ds.Vq)]
    dout = [st.out, torch.empty_like(st.out)]
    s_h2d = torch.cuda.Stream(device=dev)
    s_d2h = torch.cuda.Stream(device=dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]        # inputs b copied in
    ev_used = [torch.cuda.Event() for _ in range(2)]      # step done with inputs b / output b written
    ev_out = [torch.cuda.Event() for _ in range(2)]       # output b copied out

    def e2e_steps(n):
        for k in range(n):
            b = k & 1
            with torch.cuda.stream(s_h2d):
                if k >= 2:
                    s_h2d.wait_event(ev_used[b])
                dQ[b].copy_(hQ, non_blocking=True)
                dK[b].copy_(hK, non_blocking=True)
                dV[b].copy_(hV, non_blocking=True)
                ev_in[b].record(s_h2d)
            stream.wait_event(ev_in[b])
            if k >= 2:
                stream.wait_event(ev_out[b])
            st(dQ[b], dK[b], dV[b], ds.tau, ds.z, ds.E, ds.F, ds.e_cur, ds.e_seg, ds.seg_begin, out=dout[b])
            ev_used[b].record(stream)
            with torch.cuda.stream(s_d2h):
                s_d2h.wait_event(ev_used[b])
                hout[b].copy_(dout[b], non_blocking=True)
                ev_out[b].record(s_d2h)

    e2e_steps(args.warmup)
    torch.cuda.synchronize()
    e_start = torch.cuda.Event(enable_timing=True)
    e_end = torch.cuda.Event(enable_timing=True)
    e_start.record(s_h2d)
    e2e_steps(args.steps)
    e_end.record(s_d2h)
    torch.cuda.synchronize()
    t_e2e = max_over_ranks(e_start.elapsed_time(e_end) / 1e3, world,
                           dev if world > 1 and os.environ.get("HSA_BENCH_BACKEND", "nccl") == "nccl" else "cpu")
    e2e_value = world * shape.Lq * args.steps / t_e2e

    # work and rooflines
    peaks = load_peaks()
    pairs, inter_frac, intra_frac = exact_pairs(shape, st.selection)
    inter_h, intra_h = kept_fraction_per_head(shape, st.selection)
    w = step_work(shape)
    f_sparse = 4.0 * shape.d * pairs
    f_total = f_sparse + w["proj_flops"] + w["lin_attn_flops"]
    eff_tflops = f_total / (ms_per_step / 1e3) / 1e12
    # tensor peak: the burst figure (measured at the maximum SM clock) when the timed
    # region ran at that clock, else the sustained one (measured under the power cap)
    sm, smax = clk.get("sm_mhz"), clk.get("sm_max_mhz")
    at_max = sm is None or not smax or sm >= 0.97 * smax
    t_kind = "burst" if at_max else "sustained"
    t_peak = peaks["bf16_tflops"] if at_max else peaks["bf16_tflops_sustained"]
    host_gbs = measure_host_link(dev) if shape.host_pages else None
    # the work below is per step; a kernel launched several times a step would be rated
    # on its summed time
    kernel_work = {
        # the fused attention kernel: selected-block FLOPs of the sparse branch plus the
        # useful FLOPs of the linear branch (the split-precision extra products not counted)
        "attention_merge": ("tensor", f_sparse + w["lin_attn_flops"]),
        "linformer_proj": ("tensor", w["proj_flops"]),
        # with a host tier the timed steps gather from the HBM slots the store keeps the
        # selected pages in (host_tier reports the cold fetch over the host link)
        "gather": ("hbm", w["gather_bytes"]),
        "pool": ("hbm", w["pool_bytes"]),
        "page_scores_partial": ("hbm", w["select_pages_bytes"]),
    }
    kernels = {}
    for name, d in per_kernel.items():
        avg_ms = d["ms"] / d["launches"]
        step_ms = d["ms"] / args.steps  # the kernel's summed time a step
        entry = {"launches_per_step": d["launches"] / args.steps, "ms_per_launch": avg_ms,
                 "share": d["ms"] / sum(v["ms"] for v in per_kernel.values())}
        if name in kernel_work:
            bound, work = kernel_work[name]
            if bound == "tensor":
                ach = work / (step_ms / 1e3) / 1e12
                entry.update({"bound": "tensor", "achieved": ach, "unit": "TFLOP/s", "peak": t_peak,
                              "frac": ach / t_peak, "frac_burst": ach / peaks["bf16_tflops"],
                              "frac_sustained": ach / peaks["bf16_tflops_sustained"]})
            elif bound == "host-link":
                ach = work / (step_ms / 1e3) / 1e9  # bytes read over the host link (K and V pages)
                entry.update({"bound": "host-link", "achieved": ach, "unit": "GB/s", "peak": host_gbs,
                              "frac": ach / host_gbs if host_gbs else None})
            else:
                ach = work / (step_ms / 1e3) / 1e9
                entry.update({"bound": "hbm", "achieved": ach, "unit": "GB/s", "peak": peaks["hbm_gbs"],
                              "frac": ach / peaks["hbm_gbs"]})
        tr = traffic_of(name, shape)
        if tr is not None:
            entry["traffic"] = tr
        kernels[name] = entry
    dom = max(kernels, key=lambda k: kernels[k]["share"])
    de = kernels[dom]
    bound = de.get("bound", "hbm")
    traffic = traffic_of(dom, shape)
    peak_source = {"tensor": f"{peaks['source']} bf16 {t_kind} (median SM clock {sm} of {smax} MHz)",
                   "hbm": f"{peaks['source']} HBM copy",
                   "host-link": "pinned host-to-device copy measured in this run"}.get(bound, "")
    roofline = {"kernel": dom, "bound": bound, "achieved": de.get("achieved"), "peak": de.get("peak"),
                "unit": de.get("unit"), "frac": de.get("frac"), "traffic": traffic, "peak_source": peak_source}
    if bound == "tensor":
        roofline.update({"frac_burst": de["frac_burst"], "frac_sustained": de["frac_sustained"]})

    res = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded)",
        "config": workload_config(shape, args),
        "eff_tflops": eff_tflops,
        "selected_fraction": {"inter": inter_frac, "intra": intra_frac,
                              "inter_per_head": inter_h, "intra_per_head": intra_h},
        "roofline": roofline,
        "kernels": kernels,
        "gpu_launches": launches,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": 3 * shape.Lq * shape.H * shape.d * 2,
                "d2h_bytes_per_step": shape.Lq * shape.H * shape.d * 4,
                "copies": "pinned host buffers; H2D of step k+1 and D2H of step k-1 on copy streams beside step k"},
        "clocks": clk,
    }
    if shape.host_pages:
        res["host_tier"] = host_tier_report(ds, shape, args, host_gbs)
    res["reuse"] = reuse_report(ds, shape, args)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        heads, rows = oracle_sample_plan(shape)
        r = oracle_step_sample(ds.x, shape, oracle_summaries(ds.x, shape), heads, rows)
        res["cpu_baseline"] = {"value": shape.Lq / r["t_step"], "unit": UNIT, "cores": blas_threads(),
                               "kind": "oracle", "sample": r["sample"], "extrapolated": r["extrapolated"],
                               "timed_seconds": r["timed_seconds"], "cpu": cpu_model()}
    ds.close()
    return res if rank == 0 else None


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--workload", type=int, default=DEFAULT_WORKLOAD)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args(argv)
    args.warmup = max(3, args.warmup)
    import synth
    shape = synth.SHAPES[args.workload]
    rank, world, local = dist_setup(args.gpus)
    if args.impl == "reference":
        res = run_reference(args, shape, rank, world)
    else:
        res = run_gpu(args, shape, rank, world, local)
    if res is not None:
        print(json.dumps(res), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
