"""Benchmark of one absorbed-MLA decode step (one layer) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl mine|reference] [--config v3]

A step is the whole decode path over one batch: mla_append_absorb (the batch's new tokens into
the cache and the absorbed queries, one launch), mla_decode (split-KV attention, scheduled in
its prologue, + log-sum-exp combine) and mla_out_proj (o in the activation dtype).  The default
workload is the DeepSeek-V3-shaped single-layer decode (n_h=128, d_h=128, d_c=512, d_R=64, bf16
cache, batch 16, context 4096, s_q=1, 64-token pages).  The same line carries the other
workloads and the MHA-mode prefill (mla_prefill) under "configs".

Timing: CUDA events on the launching stream around each step, after W warm-up steps; the L2
is flushed (a 512 MiB write) before every timed step, outside the events.  Under torchrun
every rank runs its own replica (weak scaling, no collective on the data path) and the
reported time is the max over ranks.  Rank 0 prints one JSON line.

--impl reference times the fp64 CPU oracle (test infrastructure) on the host cores, on a
bounded sample of the same workload, and prints the same JSON line with "impl": "reference".
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "absorbed-MLA decode tokens/s; latent-cache GB/s & TFLOP/s vs B200 roofline"
WORKLOADS = {
    "toy": "Toy MLA layer (page-5 dims): d=1024, n_h=8, d_h=64, d_c=128, d_cq=256, d_R=32, batch 1, "
           "context 256, s_q=1, fp32",
    "v3": "DeepSeek-V3-shaped single layer decode: n_h=128, d_h=128, d_c=512, d_R=64, bf16 latent "
          "cache, batch 16, uniform context 4096, s_q=1, page 64",
    "varlen": "V3 dims, batch 64, context U[1024,16384], permuted block table, bf16",
    "long": "V3 dims, batch 4, context 131072, per-token norms LogNormal(0,0.5), bf16",
    "mtp_fp8": "V3 dims, batch 128, context 8192, s_q=2 causal, FP8 e4m3 content + bf16 RoPE key",
}
PREFILL = ("MHA-mode prefill (mla_prefill, K/V reconstructed from the latent): V3 dims n_h=128, d_h=128, "
           "d_c=512, d_R=64, bf16, 4 prompts x 4096 tokens, causal")
PREFILL_LENS = [4096] * 4
FLUSH_BYTES = 512 << 20
# DRAM bytes (read + write) per launch of the main decode kernel, from one ncu capture of the
# same workload and build (`ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum -k
# regex:decode_tc_kernel -s 2 -c 1 python bench.py --plain-steps 3 --batch 16`, caches flushed
# before the launch as in the timed loop).  None where no capture of the current kernel source
# exists: the last capture (v3: 78016512 + 2603520 bytes) predates the kernel's FP8-MMA template
# switch, so it is not reported as this build's traffic.
DECODE_TRAFFIC = {}


def make_workload(name: str, batch: int | None = None):
    from mla_latent_kv_mqa_b200 import workloads as W
    if name == "toy":
        # The toy layer's decode inputs: activations N(0, 1) (what W^DKV h, W^UQ W^DQ h, ... give
        # for h ~ N(0, 1) and nn.Linear weights ~ N(0, 1/fan_in)), W^UK, W^UV ~ N(0, 1/d_c), fp32.
        return W.make_decode(1, [256], dims=W.TOY_DIMS, act_dtype="f32", kv_dtype="f32", name="toy")
    if name == "v3":
        return W.v3_decode(B=batch or 16)
    if name == "varlen":
        return W.varlen_decode()
    if name == "long":
        return W.long_decode()
    if name == "mtp_fp8":
        return W.mtp_fp8_decode(B=batch or 128)
    raise SystemExit(f"unknown config {name}")


def max_over_ranks(values, world, device):
    """Each rank's device times -> the max over all ranks (every rank gets it); the job's time
    is the slowest replica's."""
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t]


def job_tokens(tokens_per_rank: int, world: int) -> int:
    """Query tokens one step of the whole job processes: every rank runs its own replica of the
    batch (weak scaling)."""
    return tokens_per_rank * world


def algorithmic(wl):
    """Cache bytes and FLOPs of one mla_decode over the workload (per the method's definition:
    each query row reads its visible cache rows once; 2*(d_c+d_R) + 2*d_c FLOPs per head and
    visible token)."""
    d = wl.dims
    vis = np.array([int(L) - wl.s_q + i + 1 for L in wl.seq_lens for i in range(wl.s_q)], dtype=np.int64)
    if wl.kv_dtype == "fp8":
        bpt = d.d_c + 2 * d.d_r + 4
    elif wl.kv_dtype == "f32":
        bpt = 4 * (d.d_c + d.d_r)
    else:
        bpt = 2 * (d.d_c + d.d_r)
    cache_bytes = int(wl.seq_lens.astype(np.int64).sum()) * bpt  # each cached row read once per step
    flops = int(vis.sum()) * 2 * d.n_h * ((d.d_c + d.d_r) + d.d_c)
    return cache_bytes, flops


class ClockSampler:
    """nvidia-smi samples (every 200 ms) of SM clock and throttle reasons while running, for the
    GPU whose PCI bus id is ``bus``."""
    Q = ("pci.bus_id,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, bus: int | None):
        self.bus = bus
        self.rows = []      # (arrival time, fields)
        self.error = None
        self._p = None
        self.window = None  # (t0, t1): summarise only samples that arrived in it

    def __enter__(self):
        try:
            self._p = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                                        "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True)
            self._t = threading.Thread(target=self._read, daemon=True)
            self._t.start()
        except OSError as e:
            self.error = str(e)
            self._p = None
        return self

    def _read(self):
        for line in self._p.stdout:
            r = [x.strip() for x in line.split(",")]
            if len(r) < 9:
                continue
            try:
                bus = int(r[0].split(":")[1], 16)
            except (IndexError, ValueError):
                bus = None
            if self.bus is None or bus == self.bus:
                self.rows.append((time.time(), r))

    def __exit__(self, *a):
        if self._p:
            self._p.terminate()
            try:
                _, err = self._p.communicate(timeout=5)
                if not self.rows and err:
                    self.error = err.strip()[:200]
            except subprocess.TimeoutExpired:
                self._p.kill()

    def summary(self):
        rows = [r for t, r in self.rows
                if self.window is None or self.window[0] <= t <= self.window[1]]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0,
                    "error": self.error}
        self.rows = [(0.0, r) for r in rows]
        num = lambda x: float(x) if x.replace(".", "", 1).isdigit() else None
        sm = [v for v in (num(r[1]) for _, r in self.rows) if v is not None]
        mx = [v for v in (num(r[2]) for _, r in self.rows) if v is not None]
        pw = [v for v in (num(r[3]) for _, r in self.rows) if v is not None]
        reasons = sorted({self.NAMES[i] for _, r in self.rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "power_w_max": max(pw) if pw else None, "reasons": reasons, "samples": len(self.rows),
                "window": "the last 0.5 s of the sustained warm-up load and the timed region"}


def cpu_baseline(wl, budget_s: float = 8.0, single_budget_s: float = 3.0):
    """The fp64 oracle (absorbed mode), as it stands, on a bounded sample of the workload: whole
    sequences (all heads, all visible tokens) until ``budget_s`` is spent, with the oracle's
    default host threads; then single-threaded on the first sequence, on as many heads as fit
    in about ``single_budget_s`` (scaled to all heads)."""
    import numpy as _np
    from oracle import oracle as orc
    from tests.harness import oracle_ref
    orc.build()
    threads = orc.num_threads()
    t0 = time.perf_counter()
    n_seq = 0
    for b in range(wl.B):
        oracle_ref(wl, orc, seqs=[b])
        n_seq += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    # single thread, on sequence 0's prepared inputs (the cache rows as the oracle reads them,
    # FP8 ones dequantised), so that only the decode itself is timed: one head first, then as
    # many heads as fit in the budget
    from tests.harness import oracle_cache_rows
    d = wl.dims
    cs, ks = oracle_cache_rows(wl, orc, [0])
    rows = _np.arange(wl.s_q)

    def one(nh):
        hs = _np.arange(nh)
        wsel = (hs[:, None] * d.d_h + _np.arange(d.d_h)[None, :]).reshape(-1)
        t = time.perf_counter()
        orc.decode_absorbed(wl.q_c[rows][:, hs], wl.q_r[rows][:, hs], wl.q_pos[rows], cs, ks,
                            wl.w_uk[wsel], wl.w_uv[wsel], s_q=wl.s_q, rope_base=d.rope_base)
        return time.perf_counter() - t

    orc.set_num_threads(1)
    try:
        t_one = one(1)
        nh = int(max(1, min(d.n_h, single_budget_s / max(t_one, 1e-6))))
        st = one(nh)
    finally:
        orc.set_num_threads(threads)
    st_tok = wl.s_q / (st * wl.dims.n_h / nh)  # query tokens/s with all heads, one thread
    return {"value": n_seq * wl.s_q / dt, "unit": "tokens/s", "cores": threads, "nproc": os.cpu_count(),
            "threads": threads, "kind": "oracle",
            "sample": f"{n_seq} of {wl.B} sequences, all {wl.dims.n_h} heads, fp64 absorbed mode, {dt:.1f} s",
            "single_thread": {"value": st_tok, "unit": "tokens/s",
                              "sample": f"sequence 0, {nh} of {wl.dims.n_h} heads, {st:.1f} s, scaled to all heads"}}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    wl = make_workload(args.config)
    from oracle import oracle as orc
    from tests.harness import oracle_ref
    orc.build()
    # ~150 s for the whole run whatever --steps/--warmup are; a step always finishes at least
    # one whole sequence, so a small per-step budget is still a valid sample
    budget = 150.0 / max(1, args.steps + args.warmup)
    times, toks = [], 0
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        n = 0
        for b in range(wl.B):
            oracle_ref(wl, orc, seqs=[b])
            n += 1
            if time.perf_counter() - t0 > budget:
                break
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            times.append(dt)
            toks += n * wl.s_q
    total = float(sum(times))
    value = toks / total
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / len(times),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": WORKLOADS[args.config], "sample": "per step: whole "
                                            "sequences in order until the step's CPU budget is spent"},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": orc.num_threads(), "kind": "oracle",
                             "sample": f"{toks} query tokens over {len(times)} steps, each whole sequences until "
                                       f"{budget:.2f} s were spent"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def peaks_of():
    try:
        peaks = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
        return peaks["hbm_gbs"], peaks["bf16_tflops"], "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, 1590.0, "fallback"


def step_calls(front_fused: bool, project: bool) -> str:
    front = "mla_append_absorb" if front_fused else "mla_cache_append, mla_absorb_q"
    return front + (", mla_decode_project" if project else ", mla_decode, mla_out_proj")


def fused_applies(wl) -> bool:
    """mla_decode_project runs its fused merge + projection kernel on this workload (the
    tensor-core shape: 128 heads, d_h 128, d_c 512, d_R 64, page 64, bf16 activations)."""
    d = wl.dims
    return (d.n_h, d.d_h, d.d_c, d.d_r, d.page) == (128, 128, 512, 64, 64) and wl.act_dtype == "bf16"


def measure(name, K, warmup, world, dev, clock_warmup_s, with_clock=True, project=False, separate_front=False,
            out_f32=False, fp8_mma=False):
    """Time one workload: K steps of the whole path (CUDA graph, L2 flushed before each step),
    K decode-only replays, K end-to-end steps from pinned host buffers.  Returns a dict (device
    times already reduced to the max over ranks) and the workload."""
    import torch
    import torch.distributed as dist
    from mla_latent_kv_mqa_b200 import native as N
    from tests.harness import GpuRun

    wl = make_workload(name)
    flags = N.MLA_FLAG_FP8_MMA if (fp8_mma and wl.kv_dtype == "fp8") else 0
    run = GpuRun(wl, dev=dev, flags=flags)
    run.fill_cache()
    L = run.layer
    B, s_q, T = wl.B, wl.s_q, wl.T
    # this step's new tokens: the last s_q cache rows of every sequence (rewritten every step)
    idx = np.concatenate([np.arange(wl.ctx_off[b + 1] - s_q, wl.ctx_off[b + 1]) for b in range(B)])
    tok_seq = run.tok_seq[torch.from_numpy(idx).to(dev)].contiguous()
    tok_pos = run.tok_pos[torch.from_numpy(idx).to(dev)].contiguous()
    c_new = run.c_kv[torch.from_numpy(idx).to(dev)].contiguous()
    k_new = run.k_r[torch.from_numpy(idx).to(dev)].contiguous()
    q_abs = torch.empty((T, wl.dims.n_h, wl.dims.row), dtype=run.q_c.dtype, device=dev)
    o_lat = torch.empty((T, wl.dims.n_h, wl.dims.d_c), dtype=torch.float32, device=dev)
    lse = torch.empty((T, wl.dims.n_h), dtype=torch.float32, device=dev)
    # the layer output in the activation dtype (bf16 on every V3 workload, fp32 for the toy)
    out_dt = "bf16" if (wl.act_dtype == "bf16" and not out_f32) else "f32"
    o = torch.empty((T, wl.dims.n_h, wl.dims.d_h), dtype=torch.bfloat16 if out_dt == "bf16" else torch.float32,
                    device=dev)
    L.workspace(B, s_q, run.max_seq_len)
    decode_launches = 2  # split-KV main kernel + log-sum-exp combine
    fused = fused_applies(wl) and project
    # append + absorb: one launch through mla_append_absorb where the tensor-core absorption
    # applies (the fused_applies shape), else two
    front = 1 if (fused_applies(wl) and not separate_front) else 2
    # + (main + fused merge/projection | main + combine + out_proj)
    launches_per_step = front + (2 if fused else decode_launches + 1)

    def step(_unused=None, tok=(tok_seq, tok_pos, c_new, k_new), qin=(run.q_c, run.q_r, run.q_pos), out=o):
        if separate_front:
            L.append(run.cache, tok[2], tok[3], tok[0], tok[1], run.block_table)
            L.absorb(qin[0], qin[1], qin[2], out=q_abs)
        else:
            L.append_absorb(run.cache, tok[2], tok[3], tok[0], tok[1], run.block_table, qin[0], qin[1], qin[2],
                            out=q_abs)
        if fused:
            L.decode_project(run.cache, q_abs, run.block_table, run.seq_lens, s_q, run.max_seq_len, out_dt,
                             o=out, o_lat=o_lat, lse=lse)
        else:
            L.decode(run.cache, q_abs, run.block_table, run.seq_lens, s_q, run.max_seq_len, o_lat=o_lat, lse=lse)
            L.out_proj(o_lat, out_dt, out=out)

    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.Stream(device=dev)
    # The step's inputs are packed into one pinned host buffer (256-byte aligned pieces) and one
    # device buffer, as a server would stage a batch, so a step's host-to-device traffic is one
    # copy; the calls get views into the device buffer.
    srcs = (tok_seq, tok_pos, c_new, k_new, run.q_c, run.q_r, run.q_pos)
    offs, h2d = [], 0
    for x in srcs:
        offs.append(h2d)
        h2d += (x.numel() * x.element_size() + 255) // 256 * 256
    h_pack = torch.empty(h2d, dtype=torch.uint8).pin_memory()
    d_pack = torch.empty(h2d, dtype=torch.uint8, device=dev)
    piece = lambda buf, x, off: buf[off:off + x.numel() * x.element_size()].view(x.dtype).view(x.shape)
    h_in = [piece(h_pack, x, off) for x, off in zip(srcs, offs)]
    for h, x in zip(h_in, srcs):
        h.copy_(x.cpu())
    d_in = [piece(d_pack, x, off) for x, off in zip(srcs, offs)]
    h_out = torch.empty(o.shape, dtype=o.dtype).pin_memory()
    d2h = h_out.numel() * h_out.element_size()

    def decode_only():
        L.decode(run.cache, q_abs, run.block_table, run.seq_lens, s_q, run.max_seq_len, o_lat=o_lat, lse=lse)

    def e2e_step():
        d_pack.copy_(h_pack, non_blocking=True)
        step(None, tok=tuple(d_in[:4]), qin=tuple(d_in[4:]))
        h_out.copy_(o, non_blocking=True)

    with torch.cuda.stream(stream):
        for _ in range(max(warmup, 3)):  # eager warm-up (also sets up kernel attributes)
            flush.fill_(1)
            step()
            e2e_step()
        stream.synchronize()
        if N.mla_get_last_device_error() != 0:
            raise SystemExit(f"device error during warm-up ({name})")
        g_step, g_dec, g_e2e = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_step, stream=stream):
            step()
        with torch.cuda.graph(g_dec, stream=stream):
            decode_only()
        with torch.cuda.graph(g_e2e, stream=stream):
            e2e_step()
        for _ in range(max(warmup, 3)):  # graph warm-up
            flush.fill_(2)
            g_step.replay()
            g_dec.replay()
            g_e2e.replay()
        stream.synchronize()
        mk = lambda: [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
        ev, dev_ev, e2e_ev = mk(), mk(), mk()
        bus = torch.cuda.get_device_properties(dev).pci_bus_id
        with ClockSampler(bus if with_clock else -1) as clk:
            # let the SM clock ramp up under sustained load before timing (idle boards sit far below
            # boost); the clock samples of its last half second count with the timed region's
            t_end = time.time() + max(clock_warmup_s, 0.8)
            while time.time() < t_end:
                for _ in range(20):
                    g_step.replay()
                stream.synchronize()
            if world > 1:
                dist.barrier()
            torch.cuda.synchronize()
            t_timed = time.time()
            for k in range(K):
                flush.fill_(k & 0xFF)
                ev[k][0].record(stream)
                g_step.replay()
                ev[k][1].record(stream)
                flush.fill_((k + 1) & 0xFF)
                dev_ev[k][0].record(stream)
                g_dec.replay()
                dev_ev[k][1].record(stream)
            stream.synchronize()
            if world > 1:
                dist.barrier()
            # end to end through the public API: pinned host inputs in, host result out
            for k in range(K):
                flush.fill_(k & 0xFF)
                e2e_ev[k][0].record(stream)
                g_e2e.replay()
                e2e_ev[k][1].record(stream)
                stream.synchronize()
                _ = float(h_out[0, 0, 0])  # the host reads the step's result
            clk.window = (t_timed - 0.5, time.time() + 0.15)
            time.sleep(0.15)  # the sample in flight at the end
    step_ms = sum(a.elapsed_time(b) for a, b in ev) / K
    dec_ms = sum(a.elapsed_time(b) for a, b in dev_ev) / K
    e2e_ms = sum(a.elapsed_time(b) for a, b in e2e_ev) / K
    step_ms, dec_ms, e2e_ms = max_over_ranks([step_ms, dec_ms, e2e_ms], world, dev)
    if N.mla_get_last_device_error() != 0:
        raise SystemExit(f"device error during the timed region ({name})")
    del g_step, g_dec, g_e2e
    res = dict(step_ms=step_ms, dec_ms=dec_ms, e2e_ms=e2e_ms, h2d=h2d, d2h=d2h, fused=fused,
               calls=step_calls(front == 1, fused),
               launches=(launches_per_step + decode_launches) * K, clocks=clk.summary() if with_clock else None)
    del run, flush, h_pack, d_pack, h_out
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return res, wl


def prefill_flops(wl):
    """FLOPs of one mla_prefill by the method's definition: the K and V reconstruction
    (2 T d_c n_h d_h each) and the causal attention (per head and visible (query, key) pair,
    2 (d_h + d_R) for the score and 2 d_h for the value sum)."""
    d = wl.dims
    L = wl.seq_lens.astype(np.int64)
    pairs = int((L * (L + 1) // 2).sum())
    attn = pairs * d.n_h * 2 * ((d.d_h + d.d_r) + d.d_h)
    up = 2 * 2 * wl.T * d.d_c * d.n_h * d.d_h
    return attn, up


SEQSPLIT = ("long workload (V3 dims, 4 x 131072 tokens, log-normal norms) split over 2 ranks by pages, one rank "
            "emulated on one GPU: its mla_decode over half of every sequence's pages, then mla_lse_merge_prepare and "
            "mla_lse_merge_finish (the two all-reduces between them are not in the time)")


def measure_seqsplit(K, warmup, dev, world_emul=2):
    """K timed rank-0 steps of the sequence split (CUDA graph, L2 flushed before each)."""
    import torch
    from mla_latent_kv_mqa_b200 import native as N
    from mla_latent_kv_mqa_b200 import seqsplit as S
    from tests.harness import GpuRun
    wl = make_workload("long")
    run = GpuRun(wl, dev=dev)
    run.fill_cache()
    d = run.dims
    bounds = S.page_bounds(wl.seq_lens, world_emul, wl.dims.page)
    _, n = S.token_ranges(wl.seq_lens, bounds, 0, wl.dims.page)
    bt = torch.from_numpy(S.local_block_table(wl.block_table, bounds, 0)).to(dev)
    lens = torch.from_numpy(n.astype(np.int32)).to(dev)
    rows = wl.T
    q_abs = run.layer.absorb(run.q_c, run.q_r, run.q_pos)
    o_lat = torch.empty((rows, d.n_h, d.d_c), dtype=torch.float32, device=dev)
    lse = torch.empty((rows, d.n_h), dtype=torch.float32, device=dev)
    lse_max = torch.empty_like(lse)
    acc = torch.empty(rows * d.n_h * (d.d_c + 1), dtype=torch.float32, device=dev)
    out = torch.empty_like(o_lat)
    out_lse = torch.empty_like(lse)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.Stream(device=dev)

    def step():
        run.layer.decode(run.cache, q_abs, bt, lens, 1, int(n.max()), o_lat=o_lat, lse=lse)
        lse_max.copy_(lse)  # stands in for the all-reduce(max)
        N.mla_lse_merge_prepare(rows, d.n_h, d.d_c, o_lat, lse, lse_max, acc, stream)
        N.mla_lse_merge_finish(rows, d.n_h, d.d_c, acc, lse_max, out, out_lse, stream)

    with torch.cuda.stream(stream):
        for _ in range(max(warmup, 3)):
            flush.fill_(1)
            step()
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            step()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
        for k in range(K):
            flush.fill_(k & 0xFF)
            ev[k][0].record(stream)
            g.replay()
            ev[k][1].record(stream)
        stream.synchronize()
    ms = sum(a.elapsed_time(b) for a, b in ev) / K
    if N.mla_get_last_device_error() != 0:
        raise SystemExit("device error during the sequence-split measurement")
    del g, run, flush
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return {"workload": SEQSPLIT, "ranks": world_emul, "steps": K, "rank_ms": ms,
            "tokens_per_s_if_ranks_run_together": rows / (ms * 1e-3),
            "exchange_bytes_per_allreduce": {"max": rows * d.n_h * 4, "sum": rows * d.n_h * (d.d_c + 1) * 4},
            "gpu_launches": 5 * K}


def measure_prefill(K, warmup, dev, with_clock=True, lens=None):
    """K timed mla_prefill calls (CUDA graph of the one call, L2 flushed before each)."""
    import torch
    from mla_latent_kv_mqa_b200 import native as N
    from mla_latent_kv_mqa_b200 import workloads as W
    from tests.harness import PrefillRun
    wl = W.make_prefill(9, lens or PREFILL_LENS, name="prefill")
    run = PrefillRun(wl, dev)
    o = torch.empty((wl.T, wl.dims.n_h, wl.dims.d_h), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((wl.T, wl.dims.n_h), dtype=torch.float32, device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.Stream(device=dev)
    call = lambda: run.layer.prefill(run.q_c, run.q_r, run.c_kv, run.k_r, run.cu, run.max_len, o=o, lse=lse)
    with torch.cuda.stream(stream):
        for _ in range(max(warmup, 3)):
            flush.fill_(1)
            call()
        stream.synchronize()
        if N.mla_get_last_device_error() != 0:
            raise SystemExit("device error during the prefill warm-up")
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            call()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
        bus = torch.cuda.get_device_properties(dev).pci_bus_id
        with ClockSampler(bus if with_clock else -1) as clk:
            t_end = time.time() + 0.8
            while time.time() < t_end:
                g.replay()
                stream.synchronize()
            t_timed = time.time()
            for k in range(K):
                flush.fill_(k & 0xFF)
                ev[k][0].record(stream)
                g.replay()
                ev[k][1].record(stream)
            stream.synchronize()
            clk.window = (t_timed - 0.5, time.time() + 0.15)
            time.sleep(0.15)
    ms = sum(a.elapsed_time(b) for a, b in ev) / K
    if N.mla_get_last_device_error() != 0:
        raise SystemExit("device error during the timed prefill")
    del g
    res = dict(ms=ms, launches=3 * K, clocks=clk.summary() if with_clock else None)
    del run, flush, o, lse
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return res, wl


def prefill_cpu_baseline(wl, budget_s: float = 8.0):
    """The fp64 naive-mode oracle, as it stands, on sampled prompt rows (all heads; rows drawn
    uniformly over the prompts' positions, so the mean cost per row is the workload's) until
    ``budget_s`` is spent."""
    from oracle import oracle as orc
    from tests.harness import prefill_oracle_rows
    orc.build()
    rng = np.random.default_rng(0)
    t0 = time.perf_counter()
    n = 0
    while time.perf_counter() - t0 < budget_s:
        b = int(rng.integers(0, wl.B))
        t = int(rng.integers(0, wl.seq_lens[b]))
        prefill_oracle_rows(wl, orc, [(b, t)], np.arange(wl.dims.n_h))
        n += 1
    dt = time.perf_counter() - t0
    return {"value": n / dt, "unit": "tokens/s", "cores": orc.num_threads(), "kind": "oracle",
            "sample": f"{n} prompt rows drawn uniformly, all {wl.dims.n_h} heads, fp64 naive mode, {dt:.1f} s"}


def roofline_of(wl, dec_ms):
    hbm_peak, tc_peak, src = peaks_of()
    cache_bytes, flops = algorithmic(wl)
    dec_s = dec_ms * 1e-3
    gbs = cache_bytes / dec_s / 1e9
    tfl = flops / dec_s / 1e12
    # the fp32 toy layer runs on CUDA cores: its binding peak is not the bf16 tensor one
    bound = "hbm" if cache_bytes / (hbm_peak * 1e9) >= flops / (tc_peak * 1e12) else "tensor"
    achieved, peak, unit = (gbs, hbm_peak, "GB/s") if bound == "hbm" else (tfl, tc_peak, "TFLOP/s")
    return dict(cache_bytes=cache_bytes, flops=flops, gbs=gbs, tfl=tfl, bound=bound, achieved=achieved,
                peak=peak, unit=unit, frac=achieved / peak, src=src, hbm_peak=hbm_peak, tc_peak=tc_peak)


def run_mine(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        from datetime import timedelta
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())

    from mla_latent_kv_mqa_b200 import build
    if rank == 0:
        build.build()
    if world > 1:
        dist.barrier()

    K = args.steps
    r, wl = measure(args.config, K, args.warmup, world, dev, args.clock_warmup_s, project=args.project,
                    separate_front=args.separate_front, out_f32=args.out_f32, fp8_mma=args.fp8_mma)
    rf = roofline_of(wl, r["dec_ms"])
    tokens = job_tokens(wl.T, world)
    line = None
    if rank == 0:
        dtype = {"bf16": "bf16", "f32": "f32"}.get(wl.kv_dtype, wl.kv_dtype)
        line = {
            "metric": METRIC, "value": tokens / (r["step_ms"] * 1e-3), "unit": "tokens/s", "n_gpus": world,
            "steps": K, "warmup": args.warmup, "ms_per_step": r["step_ms"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": dtype, "data": "synthetic",
            "config": {"workload": WORKLOADS[args.config], "batch_per_gpu": wl.B, "s_q": wl.s_q,
                       "context": int(wl.seq_lens.max()), "parallelism": f"replicas x{world}",
                       "l2": "flushed before every timed step (512 MiB write outside the events)",
                       "launch": "each step is one CUDA-graph replay of the calls",
                       "calls": r["calls"]},
            "decode": {"kernel": "mla_decode (tcgen05 split-KV main with in-kernel schedule + LSE combine)",
                       "ms": r["dec_ms"], "tokens_per_s": tokens / (r["dec_ms"] * 1e-3), "cache_gbs": rf["gbs"],
                       "tflops": rf["tfl"], "frac_hbm": rf["gbs"] / rf["hbm_peak"],
                       "frac_bf16": rf["tfl"] / rf["tc_peak"], "cache_bytes": rf["cache_bytes"], "flops": rf["flops"]},
            "roofline": {"bound": rf["bound"], "achieved": rf["achieved"], "peak": rf["peak"], "unit": rf["unit"],
                         "frac": rf["frac"], "traffic": DECODE_TRAFFIC.get(args.config), "peak_source": rf["src"],
                         "kernel": "mla_decode",
                         "algorithmic_per_launch": rf["cache_bytes"] if rf["bound"] == "hbm" else rf["flops"]},
            "e2e": {"value": tokens / (r["e2e_ms"] * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": r["h2d"],
                    "d2h_bytes_per_step": r["d2h"], "ms_per_step": r["e2e_ms"],
                    "how": "CUDA graph of one pinned H2D copy of the packed inputs + the step's calls + D2H of o; host reads o each step"},
            "gpu_launches": r["launches"],
            "clocks": r["clocks"],
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(wl)
    del wl
    # The other workloads, each measured the same way with fewer steps (one GPU only: under
    # torchrun every rank would hold every workload and the scaling run would take minutes).
    if world == 1 and not args.only:
        configs = {}
        k2 = max(5, K // 4)
        for name in WORKLOADS:
            if name == args.config:
                continue
            r2, wl2 = measure(name, k2, args.warmup, world, dev, 0.8, project=args.project,
                              separate_front=args.separate_front, out_f32=args.out_f32, fp8_mma=args.fp8_mma)
            rf2 = roofline_of(wl2, r2["dec_ms"])
            t2 = job_tokens(wl2.T, world)
            c = {"workload": WORKLOADS[name], "steps": k2, "step_ms": r2["step_ms"], "calls": r2["calls"],
                 "tokens_per_s": t2 / (r2["step_ms"] * 1e-3),
                 "decode_ms": r2["dec_ms"], "decode_tokens_per_s": t2 / (r2["dec_ms"] * 1e-3),
                 "cache_gbs": rf2["gbs"], "tflops": rf2["tfl"], "frac_hbm": rf2["gbs"] / rf2["hbm_peak"],
                 "frac_bf16": rf2["tfl"] / rf2["tc_peak"],
                 "roofline": {"bound": rf2["bound"], "frac": rf2["frac"], "peak": rf2["peak"], "unit": rf2["unit"],
                              "traffic": DECODE_TRAFFIC.get(name), "peak_source": rf2["src"]},
                 "e2e": {"value": t2 / (r2["e2e_ms"] * 1e-3), "unit": "tokens/s", "ms_per_step": r2["e2e_ms"],
                         "h2d_bytes_per_step": r2["h2d"], "d2h_bytes_per_step": r2["d2h"]},
                 "gpu_launches": r2["launches"], "clocks": r2["clocks"]}
            if name == "toy":
                c["roofline"]["note"] = ("fp32 layer on the CUDA-core decode kernel: launch-bound at 256 "
                                         "tokens; the fraction is reported against the bf16 peaks as is")
            if not args.no_cpu_baseline:
                c["cpu_baseline"] = cpu_baseline(wl2)
            configs[name] = c
            del wl2
        # the MHA-mode prefill (a second workload of the library, not a decode step)
        rp, wlp = measure_prefill(k2, args.warmup, dev)
        attn, up = prefill_flops(wlp)
        hbm_peak, tc_peak, src = peaks_of()
        tfl = (attn + up) / (rp["ms"] * 1e-3) / 1e12
        c = {"workload": PREFILL, "steps": k2, "ms": rp["ms"], "tokens_per_s": wlp.T / (rp["ms"] * 1e-3),
             "tflops": tfl, "flops": {"attention": attn, "kv_reconstruction": up},
             "roofline": {"bound": "tensor", "achieved": tfl, "peak": tc_peak, "unit": "TFLOP/s",
                          "frac": tfl / tc_peak, "peak_source": src,
                          "note": "whole call (prep + K/V GEMM + attention) against the dense bf16 peak"},
             "gpu_launches": rp["launches"], "clocks": rp["clocks"]}
        if not args.no_cpu_baseline:
            c["cpu_baseline"] = prefill_cpu_baseline(wlp)
        configs["prefill"] = c
        configs["seqsplit"] = measure_seqsplit(k2, args.warmup, dev)
        del wlp
        line["configs"] = configs
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def run_plain(args):
    """--plain-steps N: N eager (non-graph, untimed) steps of the workload, then exit 0.  The
    command profilers (ncu) are pointed at; --batch overrides the batch of v3 (e.g. 32, so that
    the 151 MB cache exceeds the 126 MB L2) or of mtp_fp8."""
    import torch
    from tests.harness import GpuRun
    wl = make_workload(args.config, args.batch)
    run = GpuRun(wl)
    run.fill_cache()
    for _ in range(args.plain_steps):
        if args.plain_project:
            q_abs = run.layer.absorb(run.q_c, run.q_r, run.q_pos)
            run.layer.decode_project(run.cache, q_abs, run.block_table, run.seq_lens, wl.s_q, run.max_seq_len, "f32")
        else:
            run.step()
    torch.cuda.synchronize()
    print(f"plain steps done: {args.plain_steps} x {wl.name}")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--clock-warmup-s", type=float, default=1.5)
    ap.add_argument("--impl", default="mine", choices=["mine", "reference"])
    ap.add_argument("--config", default="v3", choices=sorted(WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--only", action="store_true", help="time only --config (no per-workload block)")
    ap.add_argument("--prefill-only", action="store_true", help="time only the MHA-mode prefill workload")
    ap.add_argument("--prefill-lens", default=None, help="with --prefill-only: comma-separated prompt lengths")
    ap.add_argument("--plain-project", action="store_true",
                    help="with --plain-steps: steps through mla_decode_project")
    ap.add_argument("--fp8-mma", action="store_true",
                    help="FP8 cache: content scores on the FP8 tensor core (MLA_FLAG_FP8_MMA)")
    ap.add_argument("--out-f32", action="store_true", help="write the layer output o in fp32 (default: the "
                                                              "activation dtype)")
    ap.add_argument("--separate-front", action="store_true",
                    help="step with mla_cache_append + mla_absorb_q instead of mla_append_absorb")
    ap.add_argument("--project", action="store_true",
                    help="step with mla_decode_project (fused merge + projection) instead of mla_decode + "
                         "mla_out_proj")
    ap.add_argument("--plain-steps", type=int, default=0, help="run N untimed eager steps and exit (profiling)")
    ap.add_argument("--batch", type=int, default=None, help="with --plain-steps: batch of the v3 or mtp_fp8 workload")
    args = ap.parse_args()
    if args.prefill_only:
        import torch
        from mla_latent_kv_mqa_b200 import build
        build.build()
        torch.cuda.set_device(0)
        lens = [int(x) for x in args.prefill_lens.split(",")] if args.prefill_lens else None
        rp, wlp = measure_prefill(args.steps, args.warmup, torch.device("cuda", 0), lens=lens)
        attn, up = prefill_flops(wlp)
        print(json.dumps({"workload": PREFILL if lens is None else f"prefill, prompts {lens}",
                          "ms": rp["ms"], "tokens_per_s": wlp.T / (rp["ms"] * 1e-3),
                          "tflops": (attn + up) / (rp["ms"] * 1e-3) / 1e12, "clocks": rp["clocks"]}), flush=True)
        return
    if args.plain_steps:
        run_plain(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_mine(args)


if __name__ == "__main__":
    main()
