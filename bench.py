#!/usr/bin/env python
"""Benchmark of the positional-encoding hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ipe|reference]

One step is one pass of the whole path over one prefill request of the
large-prefill workload: a 16 x 64 x 64 video (65536 patches) through the
vision position-table interpolation and the vision 2-D rotary (one call of
the library's one-call vision entry: the two kernels run concurrently), and the
language model's interleaved multimodal RoPE on Q [131072, 24, 256] and
K [131072, 4, 256] (bf16, rotary dim 64, theta 1e7, mrope_section
[11, 11, 10]).  Inputs are seeded and synthetic, resident in HBM when the
timed region starts; every input is larger than the 126 MB L2 except the
5.3 MB position table, which a real vision tower also keeps hot.

With N > 1 (torchrun, one process per GPU) every rank runs its own request:
weak scaling with no data-path collective; the step time is the maximum over
ranks.  Rank 0 prints one JSON line.

--impl reference times the CPU oracle (double precision) on every host core
instead: one single-threaded oracle process per core, each on its own
1/16-request slice of the same workload (rank 0 only).
"""
import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time
from datetime import datetime, timedelta

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = "prefill_t131072_video"
METRIC = "Q/K MRoPE tokens/s and pos-interp patches/s; achieved HBM GB/s vs ~8 TB/s"
UNIT = "tokens/s"


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ipe", "reference"], default="ipe")
    ap.add_argument("--e2e-steps", type=int, default=50,
                    help="steps of the end-to-end (host buffers) measurement (about 22 ms each)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true", help="skip the per-variant side measurements")
    ap.add_argument("--extras-reps", type=int, default=20, help="timed repetitions of each side measurement")
    ap.add_argument("--scale-down", type=int, default=1, choices=[1, 2, 4, 8, 16],
                    help="run the step on 1/K of the tokens and video frames (profiling captures; implies "
                         "--no-e2e --no-cpu-baseline --no-extras)")
    ap.add_argument("--case", choices=sorted(CASES),
                    help="time one kernel on its own case instead of the step (profiling captures)")
    return ap.parse_args()


# ------------------------------------------------------------------ helpers


def job_time_and_value(ms_local, units_per_rank, world, reduce_max=None):
    """Step time of the job (max over ranks) and the whole-job throughput.

    Every rank runs its own request (weak scaling): the job processes
    world * units_per_rank units per step, in the time of the slowest rank.
    reduce_max(x) returns the maximum of x over ranks (None: one rank)."""
    ms = reduce_max(ms_local) if (reduce_max is not None and world > 1) else ms_local
    return ms, world * units_per_rank / (ms / 1e3)


def dist_max(value, device):
    """Maximum of a float over the ranks of the default process group."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())



def algorithmic_bytes_vision(v):
    """Interpolation bytes: table rows the samples touch, read once, plus the output."""
    import workloads as wl
    N = wl.n_patches(v)
    eb_v = 2 if v.dtype == "bf16" else 4
    G = v.grid_side
    touched = set()
    for _, h, ww in v.grid_thw:
        rows, cols = set(), set()
        for n, s in ((h, rows), (ww, cols)):
            for i in range(n):
                num = i * (G - 1)
                y0 = 0 if n == 1 else num // (n - 1)
                s.update((y0, min(y0 + 1, G - 1)))
        touched.update((y, x) for y in rows for x in cols)
    return len(touched) * v.hidden * eb_v + N * v.hidden * eb_v


def algorithmic_bytes(w):
    """Bytes each kernel must move per launch (the roofline numerator)."""
    v, t = w.vision, w.text
    import workloads as wl
    N = wl.n_patches(v)
    eb_v = 2 if v.dtype == "bf16" else 4
    rot_bytes = (t.hq + t.hk) * t.T * t.rot_dim * 2 * 2
    interp, rope = algorithmic_bytes_vision(v), 2 * N * v.heads * v.head_dim * eb_v * 2
    return {
        "vis_pos_interp": interp,
        "vis_rope2d": rope,
        "vis_pos_interp_rope2d": interp + rope,
        "mrope_apply": rot_bytes + 3 * t.T * 4,
        "mrope_cos_sin": 3 * t.T * 4 + 2 * t.T * t.rot_dim * 4,
        "apply_rotary_partial": rot_bytes + 2 * t.T * t.rot_dim * 4,
    }


def kernel_source_sha():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "interpolated_position_encoding_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def traffic_entry(kernel):
    """The committed ncu summary of `kernel` (profiles/dram_traffic.json), or
    None when the kernels changed since it was taken."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    e = d.get(WORKLOAD, {}).get(kernel)
    if not e or e.get("source_sha") != kernel_source_sha():
        return None
    return e


def dram_traffic(kernel):
    """Per-launch DRAM bytes (read + write) of `kernel` from the committed
    ncu summary, or None when the kernels changed since it was taken."""
    e = traffic_entry(kernel)
    return None if e is None else e.get("bytes_per_launch")


class ClockSampler:
    """nvidia-smi clock / throttle samples while the benchmark runs."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id):
        self.gpu_id = gpu_id
        self.proc = None
        self.file = None

    def start(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits", "-lms", "20",
                 "-i", str(self.gpu_id)], stdout=self.file, stderr=subprocess.DEVNULL)
        except (OSError, ValueError):
            self.proc = None
        return self

    def stop(self, t0, t1):
        """Summary of the samples taken between host times t0 and t1."""
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.file.flush()
        self.file.seek(0)
        rows = []
        for line in self.file.read().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                ts = datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                rows.append((ts, float(parts[2]), float(parts[3]), parts[6:10]))
            except ValueError:
                continue
        os.unlink(self.file.name)
        inside = [r for r in rows if t0 - 0.02 <= r[0] <= t1 + 0.02]
        used = inside if inside else rows
        if not used:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in used for i, v in enumerate(r[3]) if v.lower().startswith("active")})
        return {"sm_mhz": statistics.median(r[1] for r in used), "sm_max_mhz": max(r[2] for r in used),
                "reasons": reasons, "samples": len(used), "window": "timed" if inside else "whole run"}


# ------------------------------------------------------------- the oracle


def oracle_sample(w, text_tokens, frames, seed_text_offset=8192):
    """Inputs of a bounded sample of the workload for the CPU oracle: a window
    of `text_tokens` tokens (from `seed_text_offset`, through the video slices)
    and the first `frames` frames of the video."""
    import numpy as np
    import workloads as wl
    t, v = w.text, w.vision
    pos, _ = wl.build_positions(t.segments, t.merge)
    s0 = min(seed_text_offset, t.T - text_tokens)
    sl = slice(s0, s0 + text_tokens)
    key_q, key_k = wl.key_for(w.index, wl.S_Q), wl.key_for(w.index, wl.S_K)
    q = wl.normal_bf16(key_q + (s0,), (text_tokens, t.hq, t.head_dim))
    k = wl.normal_bf16(key_k + (s0,), (text_tokens, t.hk, t.head_dim))
    _, h, ww = v.grid_thw[0]
    n = frames * h * ww
    vin = {
        "table": wl.normal_bf16(wl.key_for(w.index, wl.S_TABLE), (v.grid_side ** 2, v.hidden), v.table_std),
        "q": wl.normal_bf16(wl.key_for(w.index, wl.S_QV) + (1,), (n, v.heads, v.head_dim)),
        "k": wl.normal_bf16(wl.key_for(w.index, wl.S_KV) + (1,), (n, v.heads, v.head_dim)),
    }
    f64 = lambda b: wl.bf16_bits_to_f32(b).astype(np.float64)  # noqa: E731
    return {"pos": np.ascontiguousarray(pos[:, sl]), "q": f64(q), "k": f64(k), "table": f64(vin["table"]),
            "vq": f64(vin["q"]), "vk": f64(vin["k"]), "grid": [(frames, h, ww)]}


def run_oracle(orc, w, s, text_reps=1):
    """One pass of the oracle over a sample: the text rotary on Q and K
    (text_reps times over the same window) and the vision interpolation and
    rotary on its frames."""
    t, v = w.text, w.vision
    inv = orc.rope_inv_freq(t.rot_dim, t.theta)
    for _ in range(text_reps):
        orc.mrope_apply(s["q"], s["pos"], inv, t.section, True)
        orc.mrope_apply(s["k"], s["pos"], inv, t.section, True)
    orc.vis_pos_embed_interpolate(s["table"], s["grid"], v.merge)
    orc.vis_apply_rotary(s["vq"], s["grid"], v.merge, v.theta)
    orc.vis_apply_rotary(s["vk"], s["grid"], v.merge, v.theta)


# One oracle slice: a 2048-token window rotated four times (8192 tokens of
# work) and one 64 x 64 video frame -- 1/16 of a request, with the request's
# 2 : 1 token : patch ratio.  Windows rotate through the request by worker.
SLICE_WINDOW, SLICE_REPS, SLICE_FRAMES = 2048, 4, 1
SLICE_TOKENS = SLICE_WINDOW * SLICE_REPS
SLICE_TEXT = (f"{SLICE_TOKENS} tokens (Q and K; a {SLICE_WINDOW}-token window x {SLICE_REPS}) + "
              f"{SLICE_FRAMES * 4096} patches (one 64 x 64 frame: interpolation, q and k rotary)")


def _slice_sample(w, wid):
    n_windows = (w.text.T - 8192) // SLICE_WINDOW
    return oracle_sample(w, SLICE_WINDOW, SLICE_FRAMES, seed_text_offset=8192 + (wid % n_windows) * SLICE_WINDOW)


def _oracle_worker(wid, conn):
    """An oracle process: builds its slice's inputs, reports ready, then runs
    `rounds` passes over them each time it is asked, returning the
    (monotonic) start and end of those passes."""
    import oracle
    import workloads as wl
    w = wl.WORKLOADS[WORKLOAD]
    orc = oracle.get()
    s = _slice_sample(w, wid)
    conn.send("ready")
    while True:
        rounds = conn.recv()
        if rounds is None:
            break
        t0 = time.monotonic()
        for _ in range(rounds):
            run_oracle(orc, w, s, SLICE_REPS)
        conn.send((t0, time.monotonic()))
    conn.close()


def oracle_workers():
    """Worker processes for the all-core oracle run: one per host core this
    process may use, at most 64, and at most one per 0.5 GB of available
    memory (a worker holds about 0.4 GB of float64 inputs and outputs)."""
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)
    avail = None
    try:
        with open("/proc/meminfo") as f:
            for line in f:
                if line.startswith("MemAvailable:"):
                    avail = int(line.split()[1]) * 1024
    except OSError:
        pass
    try:
        with open("/sys/fs/cgroup/memory.max") as f:
            lim = f.read().strip()
        if lim.isdigit():
            avail = min(avail or int(lim), int(lim))
    except OSError:
        pass
    n = min(cores, 64)
    if avail:
        n = min(n, max(1, int(avail // (512 << 20))))
    return max(1, n), cores


class OraclePool:
    """n oracle processes (started with spawn, one thread each), each on its
    own slice of the request; run(r) has every worker make r passes and
    returns the wall time from the first start to the last end."""

    def __init__(self, n, timeout=900):
        import multiprocessing as mp
        ctx = mp.get_context("spawn")
        self.timeout = timeout
        saved = {k: os.environ.get(k) for k in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS")}
        for k in saved:
            os.environ[k] = "1"
        self.conns, self.procs = [], []
        try:
            for i in range(n):
                a, b = ctx.Pipe()
                p = ctx.Process(target=_oracle_worker, args=(i, b), daemon=True)
                p.start()
                b.close()
                self.conns.append(a)
                self.procs.append(p)
        finally:
            for k, v in saved.items():
                if v is None:
                    os.environ.pop(k, None)
                else:
                    os.environ[k] = v
        for c in self.conns:
            if self._recv(c) != "ready":
                raise RuntimeError("oracle worker failed to start")

    def _recv(self, c):
        if not c.poll(self.timeout):
            raise RuntimeError("oracle worker did not answer")
        return c.recv()

    def run(self, rounds):
        for c in self.conns:
            c.send(rounds)
        spans = [self._recv(c) for c in self.conns]
        return max(t1 for _, t1 in spans) - min(t0 for t0, _ in spans)

    def close(self):
        for c in self.conns:
            try:
                c.send(None)
            except (BrokenPipeError, OSError):
                pass
        for p in self.procs:
            p.join(timeout=30)
            if p.is_alive():
                p.terminate()


def cpu_baseline(w, rounds=6):
    """The oracle on the host cores: every worker (one per core) runs
    `rounds` passes over its own 1/16-request slice; throughput is the tokens
    of all passes over the wall time.  The same slice on one thread in this
    process gives the single-thread figure."""
    import oracle
    orc = oracle.get()
    s = _slice_sample(w, 0)
    run_oracle(orc, w, s, SLICE_REPS)
    t0 = time.perf_counter()
    for _ in range(2):
        run_oracle(orc, w, s, SLICE_REPS)
    single = 2 * SLICE_TOKENS / (time.perf_counter() - t0)
    n, cores = oracle_workers()
    pool = OraclePool(n)
    try:
        pool.run(1)
        sec = pool.run(rounds)
    finally:
        pool.close()
    value = n * rounds * SLICE_TOKENS / sec
    return {"value": value, "unit": UNIT, "cores": n, "host_cores": cores, "kind": "oracle",
            "sample": f"{n} processes x {rounds} passes over their own slice of {SLICE_TEXT} = "
                      f"{n * rounds / 16:g} requests in {sec:.2f} s wall; tokens/s of the whole step",
            "single_thread": {"value": single, "unit": UNIT, "cores": 1,
                              "sample": f"2 passes over one slice ({SLICE_TEXT})"}}


def reference_arm(args):
    """--impl reference: the CPU oracle as the reference implementation, on
    every host core (one single-threaded process per core, each on its own
    1/16-request slice).  One step = one pass of every worker.  Rank 0
    alone runs it."""
    if int(os.environ.get("RANK", "0")) != 0:
        return
    import workloads as wl
    w = wl.WORKLOADS[WORKLOAD]
    n, cores = oracle_workers()
    pool = OraclePool(n)
    try:
        for _ in range(max(args.warmup, 0)):
            pool.run(1)
        sec = sum(pool.run(1) for _ in range(args.steps))
    finally:
        pool.close()
    value = n * SLICE_TOKENS * args.steps / sec
    sample = f"{n} processes, each one pass over its own slice of {SLICE_TEXT} per step ({n / 16:g} requests)"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec / max(args.steps, 1) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "step_sample": sample, "l2": "n/a (CPU)"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": n, "host_cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------ single-kernel cases

CASES = {
    "qk_norm_mrope": "fused QK-RMSNorm + MRoPE on text_t32768_omni (Q [32768, 32, 128], K [32768, 4, 128] bf16)",
    "rope_index": "device position table of the large-prefill request (B = 1, L = 131072, 16 video slices)",
    "mrope_decode": "decode step, B = 256, Q [256, 24, 256], K / V [256, 4, 256] bf16, norm + KV-cache write",
    "mrope_cos_sin": "cos / sin tables of the large-prefill request (T = 131072, rot 64, interleaved)",
    "vis_pos_interp_batch8": "interpolation of the batch of 8 single images (bf16 table, N = 26528)",
    "mrope_apply_prefill": "fused MRoPE of the large-prefill request (Q [131072, 24, 256], K [131072, 4, 256])",
    "mrope_apply_short": "fused MRoPE on the 4096-token prompt (text_t4096_qwen35: Q [4096, 24, 256], K [4096, 4, 256])",
    "mrope_apply_omni": "fused MRoPE on text_t32768_omni (Q [32768, 32, 128], K [32768, 4, 128] bf16, rot 128: "
                        "rows of 9 KB, rotated as two rows of half the heads)",
    "qk_norm_mrope_short": "fused QK-RMSNorm + MRoPE on the 4096-token prompt (text_t4096_qwen35)",
    "qk_norm_mrope_prefill_quarter": "fused QK-RMSNorm + MRoPE on the first 32768 tokens of the large-prefill "
                                     "request (Q [32768, 24, 256], K [32768, 4, 256] bf16, 470 MB)",
    "vis_fused_batch8": "interpolation and vision rotary in one call on the batch of 8 single images (N = 26528)",
    "vis_fused_prefill": "interpolation and vision rotary in one call on the 16 x 64 x 64 video of the large prefill",
    "vis_pos_interp_hf": "interpolation in HF rounding mode, 16 x 64 x 64 video of the large-prefill request",
    "fill_reference": "torch fill_ of the 67 MB the cos / sin kernel writes at T = 131072, rot 64 (a write-stream "
                      "reference for that kernel; not a library kernel)",
}


def run_case(args):
    """--case NAME: `--warmup` untimed and `--steps` timed calls of one
    kernel on its case (inputs resident, no L2 flush), each timed alone
    after a short GPU sleep; one JSON line."""
    import numpy as np
    import torch
    import interpolated_position_encoding_b200 as ipe
    import workloads as wl
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream()
    name = args.case
    if name == "qk_norm_mrope":
        w = wl.WORKLOADS["text_t32768_omni"]
        t = w.text
        tin = wl.text_inputs(w)
        Q = torch.from_numpy(tin["q"].view(np.int16)).view(torch.bfloat16).to(dev)
        K = torch.from_numpy(tin["k"].view(np.int16)).view(torch.bfloat16).to(dev)
        pos = torch.from_numpy(tin["positions"]).to(dev)
        wq = torch.ones(t.head_dim, dtype=torch.bfloat16, device=dev)
        inv = ipe.rope_inv_freq(t.rot_dim, t.theta)
        fn = lambda: ipe.qk_norm_mrope(Q, K, wq, wq, pos, inv, t.section, True, stream=stream)  # noqa: E731
        nbytes = (t.hq + t.hk) * t.T * t.head_dim * 2 * 2 + 3 * t.T * 4
    elif name == "rope_index":
        t = wl.WORKLOADS[WORKLOAD].text
        types, vid = _segment_types(t.segments, t.merge)
        gty, gvg = torch.from_numpy(types).to(dev), torch.from_numpy(vid).to(dev)
        B, L = types.shape
        posb = torch.empty(3, B, L, dtype=torch.int32, device=dev)
        dl = torch.empty(B, dtype=torch.int32, device=dev)
        ws = torch.empty(ipe.rope_index_workspace_bytes(B, L, 0, vid.shape[0]), dtype=torch.uint8, device=dev)
        fn = lambda: ipe.mrope_rope_index(gty, None, gvg, None, t.merge, posb, dl, ws, stream=stream)  # noqa: E731
        nbytes = B * L * 16 + B * 4
    elif name == "mrope_cos_sin":
        w = wl.WORKLOADS[WORKLOAD]
        t = w.text
        pos = torch.from_numpy(wl.text_inputs(w, with_qk=False)["positions"]).to(dev)
        inv = ipe.rope_inv_freq(t.rot_dim, t.theta)
        cos = torch.empty(t.T, t.rot_dim, dtype=torch.float32, device=dev)
        sin = torch.empty_like(cos)
        fn = lambda: ipe.mrope_cos_sin(pos, inv, t.section, True, cos, sin, stream=stream)  # noqa: E731
        nbytes = 3 * t.T * 4 + 2 * t.T * t.rot_dim * 4
    elif name in ("vis_fused_batch8", "vis_fused_prefill"):
        w = wl.WORKLOADS["vision_batch8_bf16" if name == "vis_fused_batch8" else WORKLOAD]
        v = w.vision
        vin = wl.vision_inputs(w)
        bf = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)  # noqa: E731
        table, qv, kv = bf(vin["table"]), bf(vin["q"]), bf(vin["k"])
        out = torch.empty(wl.n_patches(v), v.hidden, dtype=torch.bfloat16, device=dev)
        fn = lambda: ipe.vis_pos_interp_rope2d(table, v.grid_thw, qv, kv, v.merge, v.theta, out=out,  # noqa: E731
                                               stream=stream)
        nbytes = algorithmic_bytes_vision(v) + 2 * wl.n_patches(v) * v.heads * v.head_dim * 2 * 2
    elif name == "vis_pos_interp_hf":
        w = wl.WORKLOADS[WORKLOAD]
        v = w.vision
        table = torch.from_numpy(wl.vision_inputs(w)["table"].view(np.int16)).view(torch.bfloat16).to(dev)
        out = torch.empty(wl.n_patches(v), v.hidden, dtype=torch.bfloat16, device=dev)
        fn = lambda: ipe.vis_pos_interp(table, v.grid_thw, v.merge, out=out, stream=stream, rounding="hf")  # noqa: E731
        nbytes = algorithmic_bytes_vision(v)
    elif name == "vis_pos_interp_batch8":
        w = wl.WORKLOADS["vision_batch8_bf16"]
        v = w.vision
        table = torch.from_numpy(wl.vision_inputs(w)["table"].view(np.int16)).view(torch.bfloat16).to(dev)
        out = torch.empty(wl.n_patches(v), v.hidden, dtype=torch.bfloat16, device=dev)
        fn = lambda: ipe.vis_pos_interp(table, v.grid_thw, v.merge, out=out, stream=stream)  # noqa: E731
        nbytes = algorithmic_bytes_vision(v)
    elif name in ("mrope_apply_short", "qk_norm_mrope_short", "mrope_apply_prefill", "qk_norm_mrope_prefill_quarter",
                  "mrope_apply_omni"):
        big = name in ("mrope_apply_prefill", "qk_norm_mrope_prefill_quarter")
        w = wl.WORKLOADS["prefill_t131072_video" if big else
                         "text_t32768_omni" if name == "mrope_apply_omni" else "text_t4096_qwen35"]
        t = w.text
        tin = wl.text_inputs(w)
        T = t.T // 4 if name == "qk_norm_mrope_prefill_quarter" else t.T
        Q = torch.from_numpy(tin["q"][:T].view(np.int16)).view(torch.bfloat16).to(dev)
        K = torch.from_numpy(tin["k"][:T].view(np.int16)).view(torch.bfloat16).to(dev)
        pos = torch.from_numpy(np.ascontiguousarray(tin["positions"][:, :T])).to(dev)
        inv = ipe.rope_inv_freq(t.rot_dim, t.theta)
        if name.startswith("mrope_apply"):
            fn = lambda: ipe.mrope_apply(Q, K, pos, inv, t.section, True, stream=stream)  # noqa: E731
            nbytes = (t.hq + t.hk) * T * t.rot_dim * 2 * 2 + 3 * T * 4
        else:
            wq = torch.ones(t.head_dim, dtype=torch.bfloat16, device=dev)
            fn = lambda: ipe.qk_norm_mrope(Q, K, wq, wq, pos, inv, t.section, True, stream=stream)  # noqa: E731
            nbytes = (t.hq + t.hk) * T * t.head_dim * 2 * 2 + 3 * T * 4
    elif name == "fill_reference":
        t = wl.WORKLOADS[WORKLOAD].text
        buf = torch.empty(2 * t.T * t.rot_dim, dtype=torch.float32, device=dev)
        fn = lambda: buf.fill_(1.5)  # noqa: E731
        nbytes = buf.numel() * 4
    else:
        t = wl.WORKLOADS[WORKLOAD].text
        B, D = 256, t.head_dim
        g = torch.Generator(device=dev).manual_seed(B)
        q = torch.randn(B, t.hq, D, device=dev, generator=g).to(torch.bfloat16)
        k = torch.randn(B, t.hk, D, device=dev, generator=g).to(torch.bfloat16)
        v = torch.randn(B, t.hk, D, device=dev, generator=g).to(torch.bfloat16)
        wq = torch.ones(D, dtype=torch.bfloat16, device=dev)
        kc = torch.zeros(B * 1024, t.hk, D, dtype=torch.bfloat16, device=dev)
        vc = torch.zeros_like(kc)
        seq = torch.randint(2000, 100000, (B,), dtype=torch.int32, device=dev, generator=g)
        dl = torch.randint(-2000, 0, (B,), dtype=torch.int32, device=dev, generator=g)
        sm = torch.arange(B, device=dev, dtype=torch.int64) * 1024 + seq.long() % 1024
        inv = ipe.rope_inv_freq(t.rot_dim, t.theta)
        fn = lambda: ipe.mrope_decode(q, k, seq, inv, dl, v=v, q_weight=wq, k_weight=wq, k_cache=kc,  # noqa: E731
                                      v_cache=vc, slot_mapping=sm, stream=stream)
        nbytes = B * (t.hq + t.hk) * D * 2 * 2 + B * t.hk * D * 2 * 3 + B * 16 + 2 * D * 2
    for _ in range(max(args.warmup, 0)):
        fn()
    torch.cuda.synchronize()
    total = 0.0
    for _ in range(args.steps):
        # a short GPU sleep first, so the call is queued before its start
        # event fires and the events time the device, not the host
        torch.cuda._sleep(200_000)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        torch.cuda.synchronize()
        total += a.elapsed_time(b)
    ipe.device_status(stream)
    ms = total / max(args.steps, 1)
    peak, _ = measured_peaks()
    print(json.dumps({"case": name, "what": CASES[name], "steps": args.steps, "warmup": args.warmup, "ms": ms,
                      "alg_bytes": nbytes, "gbs": nbytes / ms / 1e6, "frac": nbytes / ms / 1e6 / peak,
                      "l2": "not flushed (inputs stay resident between launches)"}), flush=True)


# ---------------------------------------------------------------- the GPU


def main():
    args = parse_args()
    if args.impl == "reference":
        return reference_arm(args)
    if args.case:
        return run_case(args)

    import numpy as np
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.gpus != world:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE {world}: launch N > 1 with torchrun")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", device_id=dev, timeout=timedelta(seconds=300))

    import interpolated_position_encoding_b200 as ipe
    import workloads as wl

    w = wl.WORKLOADS[WORKLOAD]
    t, v = w.text, w.vision

    # ---- inputs (host, seeded; rank r > 0 shifts the stream by r)
    tin = wl.text_inputs(w)
    vin = wl.vision_inputs(w)
    if args.scale_down > 1:
        # the first 1/K of the request: its tokens and its first video frames
        import dataclasses
        f = args.scale_down
        Tn = t.T // f
        frames, gh, gw = v.grid_thw[0]
        Nn = frames // f * gh * gw
        tin = {"positions": np.ascontiguousarray(tin["positions"][:, :Tn]), "q": tin["q"][:Tn], "k": tin["k"][:Tn]}
        vin = dict(vin, q=vin["q"][:Nn], k=vin["k"][:Nn])
        t = dataclasses.replace(t, T=Tn)
        v = dataclasses.replace(v, grid_thw=[(frames // f, gh, gw)])
        w = dataclasses.replace(w, text=t, vision=v)
        args.no_e2e = args.no_cpu_baseline = args.no_extras = True
    N = wl.n_patches(v)
    if rank:
        rng = np.random.default_rng(rank)
        tin["q"] = np.roll(tin["q"], int(rng.integers(1, 1000)), axis=0)
        vin["q"] = np.roll(vin["q"], int(rng.integers(1, 1000)), axis=0)

    def dev_bf16(a):
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)

    table = dev_bf16(vin["table"])
    qv, kv = dev_bf16(vin["q"]), dev_bf16(vin["k"])
    Q, K = dev_bf16(tin["q"]), dev_bf16(tin["k"])
    pos = torch.from_numpy(tin["positions"]).to(dev)
    out = torch.empty(N, v.hidden, dtype=torch.bfloat16, device=dev)
    inv = ipe.rope_inv_freq(t.rot_dim, t.theta)
    grid = v.grid_thw
    stream = torch.cuda.current_stream()

    # the vision pair through the library's one-call entry: the interpolation
    # runs on the library's second stream beside the rotation on `stream`,
    # and `stream` waits for both, so the events on `stream` bracket both
    names = ["vis_pos_interp_rope2d", "mrope_apply"]

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        ipe.vis_pos_interp_rope2d(table, grid, qv, kv, v.merge, v.theta, out=out, stream=stream)
        if ev is not None:
            ev[1].record(stream)
        ipe.mrope_apply(Q, K, pos, inv, t.section, True, stream=stream)
        if ev is not None:
            ev[2].record(stream)

    def barrier():
        if world > 1:
            dist.barrier()

    def max_over_ranks(x):
        return x if world == 1 else dist_max(x, dev)

    props = torch.cuda.get_device_properties(dev)
    gpu_id = f"GPU-{props.uuid}" if getattr(props, "uuid", None) else str(local)
    sampler = ClockSampler(gpu_id).start()
    time.sleep(0.1)

    for _ in range(max(args.warmup, 0)):
        step()
    torch.cuda.synchronize()

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    h0 = time.time()
    start.record(stream)
    for i in range(args.steps):
        step(evs[i])
    end.record(stream)
    torch.cuda.synchronize()
    barrier()
    h1 = time.time()
    ms_step, value = job_time_and_value(start.elapsed_time(end) / args.steps, t.T, world, max_over_ranks)
    ipe.device_status(stream)          # raises if any kernel gave up a bounded wait
    kernel_ms = {n: sum(e[j].elapsed_time(e[j + 1]) for e in evs) / args.steps for j, n in enumerate(names)}
    clocks = sampler.stop(h0, h1)

    alg = algorithmic_bytes(w)
    peak, peak_src = measured_peaks()
    step_bytes = sum(alg[n] for n in names)
    kernels = {n: {"ms": kernel_ms[n], "alg_bytes": alg[n], "gbs": alg[n] / kernel_ms[n] / 1e6,
                   "frac": alg[n] / kernel_ms[n] / 1e6 / peak} for n in names}
    dom = max(names, key=lambda n: kernel_ms[n])
    tr = traffic_entry(dom) if args.scale_down == 1 else None
    roofline = {"bound": "hbm", "kernel": dom, "achieved": kernels[dom]["gbs"], "peak": peak, "unit": "GB/s",
                "frac": kernels[dom]["frac"], "traffic": None if tr is None else tr.get("bytes_per_launch"),
                "alg_bytes": alg[dom],
                "peak_source": f"{peak_src} hbm_gbs (MEASURED_PEAKS.json)" if peak_src == "measured" else
                "fallback 6650 GB/s"}
    if tr is not None and "l2_write_mb_full" in tr:
        roofline["traffic_dram_read"] = int(round(tr["dram_read_mb_full"] * 1e6))
        roofline["traffic_l2_write"] = int(round(tr["l2_write_mb_full"] * 1e6))
        roofline["traffic_note"] = ("traffic = ncu DRAM read + write per launch (1/4-size capture x 4); the DRAM writes "
                                    "undercount (lines still dirty in L2 when the kernel ends); traffic_l2_write = L2 "
                                    "write sectors x 32 B / 1.5 (calibrated on a plain fill), the bytes written")

    # ---- side measurements (after the timed region)
    extras = {}
    if not args.no_extras:
        extras = side_measurements(ipe, w, dev, stream, Q, K, pos, inv, table, qv, kv, out, alg, peak,
                                   args.extras_reps)
        extras["workloads"] = per_workload(ipe, dev, stream, peak, args.extras_reps)
        extras["next"] = next_rows(ipe, dev, stream, peak, args.extras_reps)

    # ---- end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        e2e = end_to_end(ipe, torch, w, dev, stream, vin, tin, inv, max(args.e2e_steps, 1), max_over_ranks, barrier)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w)

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD if args.scale_down == 1 else f"{WORKLOAD} at 1/{args.scale_down}",
                   "tokens_per_step": t.T, "patches_per_step": N,
                   "text": f"Q [{t.T},{t.hq},{t.head_dim}] K [{t.T},{t.hk},{t.head_dim}] bf16, rot {t.rot_dim}, "
                           f"theta {t.theta:g}, section {list(t.section)} interleaved, fused mrope_apply",
                   "vision": f"grid_thw {grid}, table [{v.grid_side ** 2},{v.hidden}] bf16, q/k [{N},{v.heads},"
                             f"{v.head_dim}] bf16, theta {v.theta:g}",
                   "l2": "no flush: every input and output but the 5.3 MB table is larger than L2",
                   "parallelism": f"dp{world} (independent requests)"},
        "patches_per_s": world * N / (ms_step / 1e3),
        "step_hbm_gbs": step_bytes / (ms_step / 1e3) / 1e9,
        "roofline": roofline,
        "kernels": kernels,
        "gpu_launches": 3 * args.steps,     # interpolation, vision rotary, fused MRoPE
        "clocks": clocks,
        "e2e": e2e,
        "cpu_baseline": cpu,
        "extras": extras,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def _time(torch, stream, fn, reps):
    fn()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(reps):
        fn()
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / reps


def side_measurements(ipe, w, dev, stream, Q, K, pos, inv, table, qv, kv, out, alg, peak, reps):
    """The unfused MRoPE (tables in HBM) and the one-launch vision variant."""
    import torch
    t, v = w.text, w.vision
    cos = torch.empty(t.T, t.rot_dim, dtype=torch.float32, device=dev)
    sin = torch.empty_like(cos)
    res = {}
    ms_cs = _time(torch, stream, lambda: ipe.mrope_cos_sin(pos, inv, t.section, True, cos, sin, stream=stream), reps)
    ms_ap = _time(torch, stream, lambda: ipe.apply_rotary_partial(Q, K, cos, sin, stream=stream), reps)
    ms_fu = _time(torch, stream, lambda: ipe.mrope_apply(Q, K, pos, inv, t.section, True, stream=stream), reps)
    for n, ms in (("mrope_cos_sin", ms_cs), ("apply_rotary_partial", ms_ap), ("mrope_apply", ms_fu)):
        res[n] = {"ms": ms, "gbs": alg[n] / ms / 1e6, "frac": alg[n] / ms / 1e6 / peak}
    res["unfused_over_fused"] = (ms_cs + ms_ap) / ms_fu
    ms_vf = _time(torch, stream, lambda: ipe.vis_pos_interp_rope2d(table, v.grid_thw, qv, kv, v.merge, v.theta,
                                                                   out=out, stream=stream), reps)
    vb = alg["vis_pos_interp"] + alg["vis_rope2d"]
    res["vis_pos_interp_rope2d"] = {"ms": ms_vf, "gbs": vb / ms_vf / 1e6, "frac": vb / ms_vf / 1e6 / peak}
    return res


def _time_flushed(torch, stream, fn, reps, flush):
    """Mean device time of fn.  Before each call (untimed) a buffer twice the
    L2 is written and then read back, so the kernel starts with its inputs out
    of L2 and with no dirty lines of the flush left to write back."""
    fn()
    total = 0.0
    for _ in range(reps):
        flush.zero_()
        flush.max()
        # keep the GPU busy while the host marshals the call, so the start
        # event is not recorded before the kernel is queued
        torch.cuda._sleep(1_000_000)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        torch.cuda.synchronize()
        total += a.elapsed_time(b)
    return total / reps


def _time_resident(torch, stream, fn, reps):
    """Mean device time of fn over back-to-back calls with nothing flushed,
    so inputs and outputs that fit stay in L2 between calls.  The stream is
    held by a device sleep while the host queues the calls, so the time is
    the GPU's, not the host's launch rate."""
    fn()
    torch.cuda.synchronize()
    torch.cuda._sleep(max(5_000_000, 400_000 * reps))   # about 0.2 ms of queueing per call
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(reps):
        fn()
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / reps


# Algorithmic bytes below which a call's tensors can stay in the 126 MB L2:
# such calls are reported both flushed and resident.
L2_RESIDENT_BYTES = 64 << 20


def per_workload(ipe, dev, stream, peak, reps):
    """Every kernel of the library on each of the five workloads (L2 flushed
    between timed calls): ms, algorithmic GB/s and fraction of the peak;
    calls small enough to stay in L2 also carry the same figures timed back
    to back without a flush ("resident")."""
    import numpy as np
    import torch
    import workloads as wl
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    res = {}

    def dev_t(a, dtype):
        if dtype == "bf16":
            return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)
        return torch.from_numpy(a).to(dev)

    def entry(ms, nbytes):
        return {"ms": ms, "gbs": nbytes / ms / 1e6, "frac": nbytes / ms / 1e6 / peak}

    def timed(fn, nbytes):
        e = entry(_time_flushed(torch, stream, fn, reps, flush), nbytes)
        if nbytes < L2_RESIDENT_BYTES:
            e["resident"] = entry(_time_resident(torch, stream, fn, reps), nbytes)
        return e

    for name, w in wl.WORKLOADS.items():
        r = {}
        if w.vision is not None:
            v = w.vision
            vin = wl.vision_inputs(w)
            N = wl.n_patches(v)
            eb = 2 if v.dtype == "bf16" else 4
            table, q, k = dev_t(vin["table"], v.dtype), dev_t(vin["q"], v.dtype), dev_t(vin["k"], v.dtype)
            out = torch.empty(N, v.hidden, dtype=table.dtype, device=dev)
            ib = algorithmic_bytes_vision(v)
            rb = 2 * N * v.heads * v.head_dim * eb * 2
            r["vis_pos_interp"] = timed(
                lambda: ipe.vis_pos_interp(table, v.grid_thw, v.merge, out=out, stream=stream), ib)
            r["vis_rope2d"] = timed(lambda: ipe.vis_rope2d(q, k, v.grid_thw, v.merge, v.theta, stream=stream), rb)
            r["vis_pos_interp_rope2d"] = timed(
                lambda: ipe.vis_pos_interp_rope2d(table, v.grid_thw, q, k, v.merge, v.theta, out=out, stream=stream),
                ib + rb)
            r["patches"] = N
        if w.text is not None:
            t = w.text
            tin = wl.text_inputs(w)
            Q, K = dev_t(tin["q"], "bf16"), dev_t(tin["k"], "bf16")
            pos = torch.from_numpy(tin["positions"]).to(dev)
            inv = ipe.rope_inv_freq(t.rot_dim, t.theta)
            cos = torch.empty(t.T, t.rot_dim, dtype=torch.float32, device=dev)
            sin = torch.empty_like(cos)
            rot = (t.hq + t.hk) * t.T * t.rot_dim * 2 * 2
            for layout in t.layouts:
                il = layout == "interleaved"
                r[f"mrope_apply/{layout}"] = timed(
                    lambda: ipe.mrope_apply(Q, K, pos, inv, t.section, il, stream=stream), rot + 3 * t.T * 4)
                r[f"mrope_cos_sin/{layout}"] = timed(
                    lambda: ipe.mrope_cos_sin(pos, inv, t.section, il, cos, sin, stream=stream),
                    3 * t.T * 4 + 2 * t.T * t.rot_dim * 4)
                r[f"apply_rotary_partial/{layout}"] = timed(
                    lambda: ipe.apply_rotary_partial(Q, K, cos, sin, stream=stream), rot + 2 * t.T * t.rot_dim * 4)
                if layout == t.layouts[0]:
                    wq = torch.ones(t.head_dim, dtype=torch.bfloat16, device=dev)
                    full = (t.hq + t.hk) * t.T * t.head_dim * 2 * 2 + 3 * t.T * 4 + 2 * t.head_dim * 2
                    r["qk_norm_mrope"] = timed(
                        lambda: ipe.qk_norm_mrope(Q, K, wq, wq, pos, inv, t.section, il, stream=stream), full)
            r["tokens"] = t.T
        res[name] = r
        torch.cuda.empty_cache()
    ipe.device_status(stream)
    return res


def _segment_types(segments, merge):
    """Token types and video-slice grids of one sample laid out from the
    workload's segments (text 0, audio 3, each vision segment a video slice)."""
    import numpy as np
    types, vid = [], []
    for kind, arg in segments:
        if kind in ("text", "audio"):
            types.append(np.full(int(arg), 0 if kind == "text" else 3, np.int32))
        else:
            t, h, w = arg
            types.append(np.full(t * (h // merge) * (w // merge), 2, np.int32))
            vid.append([t, h, w])
    return np.concatenate(types)[None], np.array(vid, np.int32).reshape(-1, 3)


def next_rows(ipe, dev, stream, peak, reps):
    """The rows beyond the path: the device position table (get_rope_index)
    and the decode step, L2 flushed between timed calls (and, when they fit
    in L2, also back to back: "resident")."""
    import numpy as np
    import torch
    import workloads as wl
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    res = {}

    def entry(ms, nbytes, **kw):
        return {"ms": ms, "gbs": nbytes / ms / 1e6, "frac": nbytes / ms / 1e6 / peak, **kw}

    def timed(fn, nbytes, **kw):
        e = entry(_time_flushed(torch, stream, fn, reps, flush), nbytes, **kw)
        if nbytes < L2_RESIDENT_BYTES:
            e["resident"] = entry(_time_resident(torch, stream, fn, reps), nbytes)
        return e

    # position table: the prefill request (B = 1) and a padded batch of 16
    t = wl.WORKLOADS[WORKLOAD].text
    types, vid = _segment_types(t.segments, t.merge)
    small = wl.WORKLOADS["text_t4096_qwen35"].text
    one, vid1 = _segment_types(small.segments, small.merge)
    B, L = 16, one.shape[1] + 300
    bt = np.zeros((B, L), np.int32)
    bm = np.zeros((B, L), np.int32)
    for b in range(B):
        bt[b, 20 * b:20 * b + one.shape[1]] = one[0]
        bm[b, 20 * b:20 * b + one.shape[1]] = 1
    for name, ty, mk, vg in (("prefill_t131072", types, None, vid), ("batch16_l4396_padded", bt, bm, np.concatenate([vid1] * B))):
        gty = torch.from_numpy(ty).to(dev)
        gmk = None if mk is None else torch.from_numpy(mk).to(dev)
        gvg = torch.from_numpy(vg).to(dev)
        Bn, Ln = ty.shape
        posb = torch.empty(3, Bn, Ln, dtype=torch.int32, device=dev)
        dl = torch.empty(Bn, dtype=torch.int32, device=dev)
        ws = torch.empty(ipe.rope_index_workspace_bytes(Bn, Ln, 0, vg.shape[0]), dtype=torch.uint8, device=dev)
        nbytes = Bn * Ln * 4 * (1 + (mk is not None) + 3) + Bn * 4
        res[f"rope_index/{name}"] = timed(
            lambda: ipe.mrope_rope_index(gty, None, gvg, gmk, t.merge, posb, dl, ws, stream=stream), nbytes,
            slots=Bn * Ln, launches=2)

    # decode step with the prefill model's heads: norm, rotation, cache write
    D, hq, hk, rot = t.head_dim, t.hq, t.hk, t.rot_dim
    inv = ipe.rope_inv_freq(rot, t.theta)
    for B in (64, 256):
        g = torch.Generator(device=dev).manual_seed(B)
        q = torch.randn(B, hq, D, device=dev, generator=g).to(torch.bfloat16)
        k = torch.randn(B, hk, D, device=dev, generator=g).to(torch.bfloat16)
        v = torch.randn(B, hk, D, device=dev, generator=g).to(torch.bfloat16)
        wq = torch.ones(D, dtype=torch.bfloat16, device=dev)
        slots_n = B * 1024
        kc = torch.zeros(slots_n, hk, D, dtype=torch.bfloat16, device=dev)
        vc = torch.zeros_like(kc)
        seq = torch.randint(2000, 100000, (B,), dtype=torch.int32, device=dev, generator=g)
        dl = torch.randint(-2000, 0, (B,), dtype=torch.int32, device=dev, generator=g)
        sm = (torch.arange(B, device=dev, dtype=torch.int64) * 1024 + seq.long() % 1024).contiguous()
        nbytes = B * (hq + hk) * D * 2 * 2 + B * hk * D * 2 * 3 + B * 16 + 2 * D * 2
        res[f"mrope_decode/b{B}_norm_cache"] = timed(
            lambda: ipe.mrope_decode(q, k, seq, inv, dl, v=v, q_weight=wq, k_weight=wq, k_cache=kc, v_cache=vc,
                                     slot_mapping=sm, stream=stream), nbytes, tokens=B, launches=1)
        del kc, vc
    # HF rounding mode: interpolation (four-corner sum) and the fused MRoPE
    for name in ("prefill_t131072_video", "vision_batch8_bf16"):
        w = wl.WORKLOADS[name]
        v = w.vision
        vin = wl.vision_inputs(w)
        table = torch.from_numpy(vin["table"].view(np.int16)).view(torch.bfloat16).to(dev)
        out = torch.empty(wl.n_patches(v), v.hidden, dtype=torch.bfloat16, device=dev)
        ms = _time_flushed(torch, stream, lambda: ipe.vis_pos_interp(table, v.grid_thw, v.merge, out=out, stream=stream,
                                                                     rounding="hf"), reps, flush)
        res[f"vis_pos_interp_hf/{name}"] = entry(ms, algorithmic_bytes_vision(v))
        del out
    w = wl.WORKLOADS[WORKLOAD]
    tin = wl.text_inputs(w)
    Q = torch.from_numpy(tin["q"].view(np.int16)).view(torch.bfloat16).to(dev)
    K = torch.from_numpy(tin["k"].view(np.int16)).view(torch.bfloat16).to(dev)
    pos = torch.from_numpy(tin["positions"]).to(dev)
    inv = ipe.rope_inv_freq(t.rot_dim, t.theta)
    ms = _time_flushed(torch, stream, lambda: ipe.mrope_apply(Q, K, pos, inv, t.section, True, stream=stream,
                                                              rounding="hf"), reps, flush)
    res[f"mrope_apply_hf/{WORKLOAD}"] = entry(ms, (t.hq + t.hk) * t.T * t.rot_dim * 2 * 2 + 3 * t.T * 4)
    del Q, K
    ipe.device_status(stream)
    torch.cuda.empty_cache()
    return res


def end_to_end(ipe, torch, w, dev, stream, vin, tin, inv, steps, max_over_ranks, barrier):
    """Same step through the C ABI's host-buffer entry points: every input
    copied in from pinned memory and every result copied back inside the
    timed region."""
    t, v = w.text, w.vision
    N = v and sum(a * b * c for a, b, c in v.grid_thw)

    def pinned_bf16(a):
        return torch.from_numpy(a.view(__import__("numpy").int16)).view(torch.bfloat16).pin_memory()

    h_in = {"table": pinned_bf16(vin["table"]), "qv": pinned_bf16(vin["q"]), "kv": pinned_bf16(vin["k"]),
            "Q": pinned_bf16(tin["q"]), "K": pinned_bf16(tin["k"]),
            "pos": torch.from_numpy(tin["positions"]).pin_memory()}
    d = {k: torch.empty_like(x, device=dev) for k, x in h_in.items()}
    out = torch.empty(N, v.hidden, dtype=torch.bfloat16, device=dev)
    h_out = {"out": torch.empty(N, v.hidden, dtype=torch.bfloat16).pin_memory(),
             "qv": torch.empty_like(h_in["qv"]).pin_memory(), "kv": torch.empty_like(h_in["kv"]).pin_memory()}
    # bytes that cross the link per step: the vision tensors whole, the text
    # Q / K rotary slices only (rotated in place on the host), positions in
    text_slices = t.T * (t.hq + t.hk) * t.rot_dim * 2
    bi = sum(h_in[k].numel() * h_in[k].element_size() for k in ("table", "qv", "kv", "pos")) + text_slices
    bo = sum(x.numel() * x.element_size() for x in h_out.values()) + text_slices

    def step():
        # the library's host-buffer entry points: chunks move in, through the
        # kernels and back, both copy directions overlapping; the last call
        # joins `stream`, so the step ends when every result is in host memory
        ipe.vis_pos_interp_host(h_in["table"], v.grid_thw, h_out["out"], d["table"], out, v.merge,
                                chunk_rows=16384, join=False, stream=stream)
        ipe.vis_rope2d_host(h_in["qv"], h_in["kv"], v.grid_thw, d["qv"], d["kv"], v.merge, v.theta, h_out["qv"],
                            h_out["kv"], chunk_rows=8192, join=False, stream=stream)
        # in place on the host Q / K: only the rotary slices cross the link
        ipe.mrope_apply_host(h_in["Q"], h_in["K"], h_in["pos"], inv, t.section, True, d["Q"], d["K"], d["pos"],
                             chunk_tokens=4096, join=True, stream=stream)

    step()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    a.record(stream)
    for _ in range(steps):
        step()
    b.record(stream)
    torch.cuda.synchronize()
    barrier()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    ms, value = job_time_and_value(a.elapsed_time(b) / steps, t.T, world, max_over_ranks)
    return {"value": value, "unit": UNIT, "h2d_bytes_per_step": bi, "d2h_bytes_per_step": bo,
            "ms_per_step": ms, "steps": steps}


if __name__ == "__main__":
    main()
