"""Benchmark of split-value-cache decode attention (and the prefill chunk).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl lrkv|reference] [--workload NAME]

Default workload (the headline): the largest single-GPU decode workload, the
Qwen3-1.7B-shaped long-context case (28 layers, 16 query / 8 KV heads, d = 128,
eight agents in BaseShared mode at r = 16, 4 sessions, 65536 shared tokens in
64-token pages with a random page order, offsets drawn in [32768, 65536)).  One
step = one decode query per (session, agent) through the attention of all 28
layers (28 launches of the decode kernel, captured once in a CUDA graph and
replayed).  Inputs are synthetic (seeded N(0, 1) draws of the model's shapes)
and resident in HBM; each layer has its own buffers, so a step streams 30 GB
(> L2) and no L2 flush is needed between steps.

The same JSON line carries, under ``decode_workloads``, the other decode
workloads timed the same way (the Qwen2.5-Coder-1.5B case and each context
length of the Qwen3-1.7B sweep), and under ``prefill`` the append + causal
prefill-chunk step, under ``sharing`` the shared / non-shared / full-shared
comparison.

Prints ONE JSON line (rank 0).  Under torchrun each rank runs the same
workload on its own data (weak scaling, no collective on the data path); the
step time is the max over ranks.

``--impl reference`` times the fp64 CPU oracle on the host cores instead, on
a bounded sample of the same workload (the one other place this script runs
the oracle besides the cpu_baseline leg).
"""

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from workloads import CONFIGS, make_decode_inputs, make_prefill_inputs  # noqa: E402

METRIC = "LoRA-split KV attention: decode queries/s, HBM GB/s vs ~8 TB/s peak"
NOMINAL_HBM_GBS = 8000.0        # B200 HBM3e, nominal
NOMINAL_BF16_TFLOPS = 2250.0    # B200 dense bf16, nominal
UNIT = "queries/s"
BF16 = 2


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            pk = json.load(f)
        return float(pk["hbm_gbs"]), float(pk["bf16_tflops"]), float(pk["bf16_tflops_sustained"]), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


# ---------------------------------------------------------------------------
# DRAM traffic from the committed ncu summaries
# ---------------------------------------------------------------------------

# Sources that decide what a kernel reads and writes.  A summary under
# profiles/ records their sha256 at capture time; its DRAM bytes are reported
# only while the sources still hash the same (else the counters are stale).
KERNEL_SOURCES = {
    "decode_kernel": ["decode.cu", "common.cuh", "lrkv_internal.h", "lrkv_api.cu"],
    "prefill_kernel": ["prefill.cu", "prefill.h", "common.cuh", "lrkv_internal.h", "lrkv_api.cu"],
}


def kernel_sources_sha256(kernel):
    """sha256 of the kernel's sources with their comments removed and whitespace
    folded (a change of comments or layout alone does not change what the
    kernel reads and writes)."""
    import hashlib
    import re
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "lora_shared_kv_b200", "csrc", name)) as f:
            src = f.read()
        src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
        src = re.sub(r"//[^\n]*", " ", src)
        h.update(" ".join(src.split()).encode())  # and with whitespace runs folded
    return h.hexdigest()


def profiled_traffic(kernel, workload):
    """DRAM bytes (read + write) per launch of `kernel` on `workload` from
    profiles/<kernel>__<workload>.md, or None when there is no summary or the
    kernel's sources changed since it was taken."""
    path = os.path.join(ROOT, "profiles", f"{kernel}__{workload}.md")
    try:
        with open(path) as f:
            text = f.read()
    except OSError:
        return None
    fields = {}
    for line in text.splitlines():
        line = line.strip().lstrip("-* ").strip()
        if ":" in line:
            k, v = line.split(":", 1)
            fields[k.strip().strip("`")] = v.strip().strip("`")
    try:
        if fields.get("sources_sha256") != kernel_sources_sha256(kernel):
            return None
        return int(fields["dram_bytes_per_launch"])
    except (KeyError, ValueError, OSError):
        return None


# ---------------------------------------------------------------------------
# algorithmic bytes
# ---------------------------------------------------------------------------

def decode_layer_bytes(cfg, offsets_cpu):
    """Bytes one decode launch must move: K and V once for all agents, the U rows
    at or past each offset (once per U cache; shared by the KV heads), q, out, B,
    and the page table."""
    S, N, Hq, Hkv, d, r, L = cfg.S, cfg.N, cfg.Hq, cfg.Hkv, cfg.d, cfg.r, cfg.L
    kv = 2 * S * Hkv * L * d * BF16
    offs = np.clip(offsets_cpu.numpy().astype(np.int64), 0, L)
    if cfg.mode == 0:
        u_rows = int(np.sum(L - offs))
    else:
        u_rows = int(np.sum(L - offs.min(axis=1)))
    u = u_rows * r * BF16
    qo = 2 * S * N * Hq * d * BF16
    b = N * r * Hkv * d * BF16
    pt = S * math.ceil(L / cfg.page_size) * 4 if cfg.paged else 0
    return kv + u + qo + b + pt


def shard_layer_bytes(cfg, offsets_cpu, blocks):
    """decode_layer_bytes for the (session_begin, session_count, head_begin,
    head_count) blocks of one rank: each block reads the K/V of its heads, the
    U rows of its sessions (U is shared by the heads, so every block that holds
    a session reads them), its heads' q, out and B columns, and its page-table rows."""
    N, Hq, Hkv, d, r, L = cfg.N, cfg.Hq, cfg.Hkv, cfg.d, cfg.r, cfg.L
    G = Hq // Hkv
    offs = np.clip(offsets_cpu.numpy().astype(np.int64), 0, L)
    total = 0
    for (s0, ns, g0, ng) in blocks:
        o = offs[s0:s0 + ns]
        u_rows = int(np.sum(L - o)) if cfg.mode == 0 else int(np.sum(L - o.min(axis=1)))
        total += 2 * ns * ng * L * d * BF16 + u_rows * r * BF16 + 2 * ns * N * ng * G * d * BF16
        total += N * r * ng * d * BF16 + (ns * math.ceil(L / cfg.page_size) * 4 if cfg.paged else 0)
    return total


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        self.out = []
        self.dev = device_index

    def start(self):
        try:
            uuid = str(torch.cuda.get_device_properties(self.dev).uuid)
            sel = ["-i", uuid if uuid.startswith("GPU-") else "GPU-" + uuid]
        except Exception:
            sel = []
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "10"] + sel, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out = ""
        rows = [ln.split(",") for ln in out.strip().splitlines() if ln.count(",") >= 8]
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                smax = float(r[2])
                for i, nm in enumerate(names):
                    if r[5 + i].strip().lower() == "active":
                        reasons.add(nm)
            except ValueError:
                continue
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# decode workload on the GPU
# ---------------------------------------------------------------------------

class DecodeRunner:
    def __init__(self, cfg, device, seed_offset=0):
        import lora_shared_kv_b200 as lrkv
        self.lrkv = lrkv
        self.cfg = cfg
        self.dev = device
        from workloads.gen import seed_for
        self.inp = make_decode_inputs(cfg, device=device, seed=seed_for(cfg) + seed_offset)
        c = cfg
        self.prob = lrkv.make_problem(c.S, c.N, c.Hq, c.Hkv, c.d, c.r, c.mode)
        nws = lrkv.lrkv_decode_workspace_bytes(self.prob, c.L)
        self.ws = torch.zeros(nws, dtype=torch.uint8, device=device)
        self.outs = [torch.empty((c.S, c.N, c.Hq, c.d), dtype=torch.bfloat16, device=device) for _ in self.inp.layers]
        self.kvs = []
        self.uvs = []
        for lay in self.inp.layers:
            if c.paged:
                self.kvs.append(lrkv.kv_view_paged(lay.k, lay.v, lay.page_table))
            else:
                self.kvs.append(lrkv.kv_view_dense(lay.k, lay.v))
            self.uvs.append(lrkv.u_view(lay.u))
        self.graph = None
        self.blocks = None

    def set_shard(self, blocks):
        """Serve only the given (session_begin, session_count, head_begin, head_count)
        blocks of every layer (lrkv_attn_decode_kv_heads on views of the shard)."""
        lrkv, c, inp = self.lrkv, self.cfg, self.inp
        self.blocks = []
        ws_bytes = 0
        for (s0, ns, g0, ng) in blocks:
            prob = lrkv.make_problem(ns, c.N, c.Hq, c.Hkv, c.d, c.r, c.mode)
            ws_bytes = max(ws_bytes, lrkv.lrkv_decode_kv_heads_workspace_bytes(prob, ng, c.L))
            per_layer = []
            for lay in inp.layers:
                if c.paged:
                    kv = lrkv.kv_view_paged(lay.k[:, g0:g0 + ng], lay.v[:, g0:g0 + ng], lay.page_table[s0:s0 + ns])
                else:
                    kv = lrkv.kv_view_dense(lay.k[s0:s0 + ns, g0:g0 + ng], lay.v[s0:s0 + ns, g0:g0 + ng])
                per_layer.append((kv, lrkv.u_view(lay.u[s0:s0 + ns])))
            self.blocks.append((s0, ns, g0, ng, prob, per_layer))
        self.ws = torch.zeros(ws_bytes, dtype=torch.uint8, device=self.dev)
        self.queries_served = c.S * c.N * sum(ns * ng for (_, ns, _, ng, _, _) in self.blocks) // (c.S * c.Hkv)

    def layer(self, li, q, out, stream=None):
        """Decode attention of layer li (this rank's blocks of it, when sharded)."""
        lrkv, c, inp = self.lrkv, self.cfg, self.inp
        lay = inp.layers[li]
        if self.blocks is None:
            lrkv.lrkv_attn_decode(self.prob, q, self.kvs[li], inp.seq_lens, c.L, self.uvs[li], lay.b,
                                  inp.offsets, out, self.ws, stream=stream)
            return
        for (s0, ns, g0, ng, prob, per_layer) in self.blocks:
            kv, uv = per_layer[li]
            lrkv.lrkv_attn_decode_kv_heads(prob, g0, ng, q[s0:s0 + ns], kv, inp.seq_lens[s0:s0 + ns], c.L, uv,
                                           lay.b, inp.offsets[s0:s0 + ns], out[s0:s0 + ns], self.ws,
                                           stream=stream)

    def step_eager(self, qs=None, outs=None, stream=None):
        for li, lay in enumerate(self.inp.layers):
            self.layer(li, lay.q if qs is None else qs[li], self.outs[li] if outs is None else outs[li], stream)

    def capture(self):
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            self.step_eager()
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            self.step_eager()
        torch.cuda.synchronize()

    def step(self):
        self.graph.replay()

    @property
    def launches_per_step(self):
        return len(self.inp.layers) * (1 if self.blocks is None else len(self.blocks))

    def layer_bytes(self):
        """Algorithmic bytes of one layer's launches on this rank."""
        if self.blocks is None:
            return decode_layer_bytes(self.cfg, self.inp.offsets.cpu())
        return shard_layer_bytes(self.cfg, self.inp.offsets.cpu(), [b[:4] for b in self.blocks])


# ---------------------------------------------------------------------------
# ranks: one process per GPU, each with its own sessions (weak scaling)
# ---------------------------------------------------------------------------

def rank_seed_offset(rank: int) -> int:
    """Every rank draws its own sessions: the seed moves by a prime per rank."""
    return 7919 * rank


def kv_head_shard_plan(S: int, Hkv: int, world: int):
    """Split one workload's (session, KV head) pairs over `world` ranks.

    The pairs are taken in session-major order and rank r gets the contiguous
    range [r U / world, (r + 1) U / world) of the U = S * Hkv pairs, written as
    blocks (session_begin, session_count, head_begin, head_count) that one
    lrkv_attn_decode_kv_heads call each serves (whole sessions, or a head range
    of one session).  Every pair lands in exactly one block of one rank; the
    ranks exchange nothing (each KV head reads only its own K/V and B columns)."""
    U = S * Hkv
    plan = []
    for r in range(world):
        lo, hi = r * U // world, (r + 1) * U // world
        blocks = []
        u = lo
        while u < hi:
            s, g = divmod(u, Hkv)
            if g == 0 and hi - u >= Hkv:
                n_s = (hi - u) // Hkv
                blocks.append((s, n_s, 0, Hkv))
                u += n_s * Hkv
            else:
                cnt = min(Hkv - g, hi - u)
                blocks.append((s, 1, g, cnt))
                u += cnt
        plan.append(blocks)
    return plan


def max_over_ranks(x: float, device=None) -> float:
    """The slowest rank's time (a timing reduction only, never on the data path)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: float, world: int, ms_max: float) -> float:
    """Whole-job units per second: all ranks' units over the slowest rank's time."""
    return units_per_rank * world / (ms_max * 1e-3)


def _timed(fn, steps, warmup, sync_all):
    for _ in range(warmup):
        fn()
    sync_all()
    st = torch.cuda.current_stream()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for _ in range(steps):
        fn()
    e1.record(st)
    e1.synchronize()
    sync_all()
    return e0.elapsed_time(e1)


def cpu_sample_layers(cfg, n_layers):
    """Layers the CPU baseline times per session: all of them, or for the long
    contexts (where one session through every layer would take minutes of fp64
    work) the first, middle and last layer, with the time scaled by
    n_layers / 3 (reported as extrapolated)."""
    if cfg.L >= 32768 and n_layers > 3:
        return [0, n_layers // 2, n_layers - 1]
    return list(range(n_layers))


def cpu_baseline_decode(runner, min_seconds=10.0, max_seconds=25.0):
    """fp64 oracle on the host cores: session after session, each through the
    sampled layers (cpu_sample_layers), until at least min_seconds of oracle
    time (at most max_seconds).  Only the oracle calls are timed, not the
    copies of the inputs to the host."""
    import oracle
    from threadpoolctl import threadpool_info
    cfg, inp = runner.cfg, runner.inp
    nl = len(inp.layers)
    layers = cpu_sample_layers(cfg, nl)
    cores = len(os.sched_getaffinity(0))
    blas_threads = max([d.get("num_threads", 1) for d in threadpool_info()] + [1])
    dt = 0.0
    done_layers = 0
    sessions = 0
    for s in range(cfg.S):
        offs = inp.offsets[s:s + 1].cpu()
        sl = inp.seq_lens[s:s + 1].cpu()
        for li in layers:
            lay = inp.layers[li]
            q, u, b = lay.q[s:s + 1].cpu(), lay.u[s:s + 1].cpu(), lay.b.cpu()
            if cfg.paged:  # this session's pages, in logical order
                pt = lay.page_table[s].long()
                k, v = lay.k[pt].cpu(), lay.v[pt].cpu()
                table = torch.arange(pt.numel(), dtype=torch.int32).view(1, -1)
            else:
                k, v, table = lay.k[s:s + 1].cpu(), lay.v[s:s + 1].cpu(), None
            t0 = time.perf_counter()
            oracle.decode(q, k, v, u, b, offs, sl, cfg.mode, page_table=table)
            dt += time.perf_counter() - t0
            done_layers += 1
            if dt > max_seconds:
                break
        sessions += 1
        if dt > min_seconds:
            break
    # one query = one (session, agent) through all nl layers; the sampled layers stand for all of them
    queries = cfg.N * done_layers / len(layers)
    t_all = dt * nl / len(layers)
    extrap = len(layers) < nl
    sample = (f"{sessions} session(s) x layers {layers if extrap else f'0..{nl - 1}'} "
              f"({done_layers} session-layers, {queries:.2f} queries), fp64 numpy, {dt:.1f} s of oracle time")
    if extrap:
        sample += f"; extrapolated to all {nl} layers (time x {nl}/{len(layers)})"
    sample += f"; {cores} cores visible, BLAS threads {blas_threads}"
    return {"value": queries / t_all, "unit": UNIT, "cores": min(cores, blas_threads) if blas_threads else cores,
            "kind": "oracle", "extrapolated": extrap, "sample": sample}


def run_e2e(runner, steps, warmup, sync_all):
    """Public API with host buffers.  Per step every layer's q is copied from
    pinned host memory and every layer's output back, each on its own copy
    stream and ordered against the decode calls by events, so layer l's copies
    overlap the neighbouring layers' attention; the step ends when the last
    output has landed on the host."""
    c = runner.cfg
    nl = len(runner.inp.layers)
    lrkv = runner.lrkv
    inp = runner.inp
    q_host = torch.stack([lay.q for lay in inp.layers]).cpu().pin_memory()
    out_host = torch.empty((nl, c.S, c.N, c.Hq, c.d), dtype=torch.bfloat16).pin_memory()
    q_dev = torch.empty_like(q_host, device=runner.dev)
    out_dev = torch.empty_like(out_host, device=runner.dev)
    comp = torch.cuda.current_stream(runner.dev)
    h2d = torch.cuda.Stream(runner.dev)
    d2h = torch.cuda.Stream(runner.dev)
    ev_in = [torch.cuda.Event() for _ in range(nl)]
    ev_out = [torch.cuda.Event() for _ in range(nl)]

    def step():
        h2d.wait_stream(comp)  # the previous step no longer reads q_dev
        with torch.cuda.stream(h2d):
            for li in range(nl):
                q_dev[li].copy_(q_host[li], non_blocking=True)
                ev_in[li].record(h2d)
        for li in range(nl):
            comp.wait_event(ev_in[li])
            runner.layer(li, q_dev[li], out_dev[li])
            ev_out[li].record(comp)
        with torch.cuda.stream(d2h):
            for li in range(nl):
                d2h.wait_event(ev_out[li])
                out_host[li].copy_(out_dev[li], non_blocking=True)
        comp.wait_stream(d2h)

    ms = _timed(step, steps, warmup, sync_all)
    return ms / steps, q_host.numel() * 2, out_host.numel() * 2


def _eager_ms(fn, steps, warmup):
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        fn()
    e1.record()
    e1.synchronize()
    return e0.elapsed_time(e1) / steps


def sharing_comparison(runner, max_bytes=40e9, steps=10, warmup=3, return_outputs=False):
    """The pages' comparison of cache sharing, on the same decode kernel.

    - shared: the split value cache (base K/V once for all agents, rank-r U_i);
    - non-shared: every agent holds its own K and its own materialised
      V_i = V_base + Umask_i B_i (N times the K/V bytes), run as S*N single-agent
      sessions with B = 0;
    - full-shared: the base K/V alone, the adapter's value term dropped (no U
      read, B = 0): the approximation the split cache avoids.
    Times are per layer (eager launches) over the first layers whose non-shared
    copies fit in max_bytes; the non-shared outputs are checked against the
    shared ones (they differ only by the bf16 rounding of V_i).  With
    return_outputs, also returns every arm's outputs per timed layer
    ({"shared", "non_shared", "full_shared"}: lists of [S, N, Hq, d] tensors)."""
    lrkv, c, inp, dev = runner.lrkv, runner.cfg, runner.inp, runner.dev
    S, N, Hq, Hkv, d, r, L = c.S, c.N, c.Hq, c.Hkv, c.d, c.r, c.L
    per_layer_ns = 2 * S * N * Hkv * L * d * BF16
    nl = max(1, min(len(inp.layers), int(max_bytes // per_layer_ns)))
    keep = torch.arange(L, device=dev)[None, None, :] >= inp.offsets[:, :, None].long()  # [S, N, L]
    prob_ns = lrkv.make_problem(S * N, 1, Hq, Hkv, d, r, lrkv.BASE_SHARED)
    ws_ns = torch.zeros(lrkv.lrkv_decode_workspace_bytes(prob_ns, L), dtype=torch.uint8, device=dev)
    u_none = torch.zeros((S * N, 1, L, r), dtype=torch.bfloat16, device=dev)
    uv_none = lrkv.u_view(u_none)
    b_zero = torch.zeros((1, r, Hkv * d), dtype=torch.bfloat16, device=dev)
    offs_ns = torch.full((S * N, 1), L, dtype=torch.int32, device=dev)
    offs_full = torch.full_like(inp.offsets, L)
    b_zero_n = torch.zeros((N, r, Hkv * d), dtype=torch.bfloat16, device=dev)
    outs_full = [torch.empty_like(runner.outs[li]) for li in range(nl)]
    ns = []
    for li in range(nl):
        lay = inp.layers[li]
        if c.paged:
            pt = lay.page_table.long()
            k = lay.k[pt].permute(0, 2, 1, 3, 4).reshape(S, Hkv, L, d)
            v = lay.v[pt].permute(0, 2, 1, 3, 4).reshape(S, Hkv, L, d)
        else:
            k, v = lay.k, lay.v
        k_ns = k.repeat_interleave(N, dim=0).contiguous()
        v_ns = torch.empty_like(k_ns)
        for i in range(N):
            ui = lay.u[:, i if c.mode == 0 else 0].float() * keep[:, i, :, None]          # [S, L, r]
            vi = v.float() + torch.einsum("slr,rgd->sgld", ui, lay.b[i].float().view(r, Hkv, d))
            v_ns[i::N] = vi.to(torch.bfloat16)
        ns.append((k_ns, v_ns, lay.q.reshape(S * N, 1, Hq, d).contiguous(),
                   torch.empty((S * N, 1, Hq, d), dtype=torch.bfloat16, device=dev)))
    kv_ns = [lrkv.kv_view_dense(k_ns, v_ns) for k_ns, v_ns, _, _ in ns]

    def run_shared():
        for li in range(nl):
            lay = inp.layers[li]
            lrkv.lrkv_attn_decode(runner.prob, lay.q, runner.kvs[li], inp.seq_lens, L, runner.uvs[li], lay.b,
                                  inp.offsets, runner.outs[li], runner.ws)

    def run_full_shared():
        for li in range(nl):
            lay = inp.layers[li]
            lrkv.lrkv_attn_decode(runner.prob, lay.q, runner.kvs[li], inp.seq_lens, L, runner.uvs[li], b_zero_n,
                                  offs_full, outs_full[li], runner.ws)

    seq_ns = inp.seq_lens.repeat_interleave(N)

    def run_non_shared():
        for li in range(nl):
            _, _, q_ns, o_ns = ns[li]
            lrkv.lrkv_attn_decode(prob_ns, q_ns, kv_ns[li], seq_ns, L, uv_none, b_zero, offs_ns, o_ns, ws_ns)

    t_ns = _eager_ms(run_non_shared, steps, warmup) / nl
    t_full = _eager_ms(run_full_shared, steps, warmup) / nl
    t_sh = _eager_ms(run_shared, steps, warmup) / nl  # leaves the shared outputs in runner.outs
    torch.cuda.synchronize()
    max_abs = max(float((runner.outs[li].float() - ns[li][3].view(S, N, Hq, d).float()).abs().max())
                  for li in range(nl))
    kv_shared = 2 * S * Hkv * L * d * BF16 + S * c.n_u * L * r * BF16
    out = {"workload": c.name, "layers_timed": nl, "ms_per_layer_shared": t_sh,
           "ms_per_layer_non_shared": t_ns, "ms_per_layer_full_shared": t_full,
           "speedup_shared_vs_non_shared": t_ns / t_sh,
           "cache_bytes_per_layer_shared": kv_shared, "cache_bytes_per_layer_non_shared": per_layer_ns,
           "max_abs_non_shared_vs_shared": max_abs,
           "note": "eager launches; non-shared = per-agent K and materialised V_i, B = 0; full-shared = base K/V only"}
    arms = None
    if return_outputs:
        arms = {"shared": [runner.outs[li].clone() for li in range(nl)],
                "non_shared": [ns[li][3].view(S, N, Hq, d).clone() for li in range(nl)],
                "full_shared": outs_full}
    del ns, kv_ns
    torch.cuda.empty_cache()
    return (out, arms) if return_outputs else out


def value_projection_timing(cfg, inp, prob, device, steps=20, warmup=5):
    """The chunk's value projection [V_base | U_1..U_n] = X [W0_v | A_1..A_n]
    into the caches (the step before the attention): median time and TFLOP/s.
    The weights are synthetic draws of the model's shapes."""
    import lora_shared_kv_b200 as lrkv
    g = torch.Generator(device=device)
    g.manual_seed(4242)
    ncols = cfg.Hkv * cfg.d + cfg.n_u * cfg.r
    w = (torch.randn((cfg.Dm, ncols), generator=g, device=device) * cfg.Dm ** -0.5).to(torch.bfloat16)
    v = torch.empty_like(inp.v)
    kv = lrkv.kv_view_dense(inp.k, v)
    u = torch.empty_like(inp.u)
    ws = torch.zeros(256, dtype=torch.uint8, device=device)
    rows = inp.v.shape[2]

    def step():
        lrkv.lrkv_value_projection(prob, inp.x, w, kv, rows, u, 0, cfg.L0, ws)

    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=device)
    times = []
    for i in range(warmup + steps):
        flush.zero_()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        step()
        e1.record()
        e1.synchronize()
        if i >= warmup:
            times.append(e0.elapsed_time(e1))
    ms = statistics.median(times)
    flops = 2.0 * cfg.T * cfg.Dm * ncols
    return {"ms": ms, "tflops": flops / (ms * 1e-3) / 1e12, "flops": flops,
            "shape": f"X [{cfg.T}, {cfg.Dm}] x W [{cfg.Dm}, {ncols}]"}


def bench_prefill(device, steps=20, warmup=5):
    """Prefill chunk workload: append the chunk's U rows, then the causal chunk
    attention for 4 agents (one layer).  Returns a dict, or None if unavailable."""
    import lora_shared_kv_b200 as lrkv
    cfg = CONFIGS["cfg4"]
    inp = make_prefill_inputs(cfg, device=device)
    prob = lrkv.make_problem(1, cfg.N, cfg.Hq, cfg.Hkv, cfg.d, cfg.r, cfg.mode)
    kv = lrkv.kv_view_dense(inp.k, inp.v)
    uv = lrkv.u_view(inp.u)
    nws = lrkv.lrkv_prefill_workspace_bytes(prob, cfg.L0, cfg.T)
    ws = torch.zeros(max(nws, 256), dtype=torch.uint8, device=device)
    out = torch.empty((cfg.N, cfg.T, cfg.Hq, cfg.d), dtype=torch.bfloat16, device=device)

    def append():
        lrkv.lrkv_append_lr_cache(inp.x, inp.a_down, inp.u, session=0, start_row=cfg.L0, uview=uv)

    def chunk():
        lrkv.lrkv_attn_prefill_chunk(prob, inp.q, kv, 0, cfg.L0, cfg.T, uv, inp.b, inp.offsets, out, ws)

    def step():
        append()
        chunk()

    try:
        step()
    except Exception as e:  # noqa: BLE001
        return {"status": f"unavailable: {e}"}
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=device)

    def median_ms(fn):
        times = []
        for i in range(warmup + steps):
            flush.zero_()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            e1.synchronize()
            if i >= warmup:
                times.append(e0.elapsed_time(e1))
        return statistics.median(times)

    ms = median_ms(step)
    append_ms, chunk_ms = median_ms(append), median_ms(chunk)
    vproj = value_projection_timing(cfg, inp, prob, device)
    keys = cfg.T * cfg.L0 + cfg.T * (cfg.T + 1) // 2
    rows = cfg.N * cfg.Hq
    flops = 2.0 * rows * keys * cfg.d * 2 + 2.0 * rows * keys * cfg.r + 2.0 * rows * cfg.T * cfg.r * cfg.d
    flops += 2.0 * cfg.N * cfg.T * cfg.Dm * cfg.r
    _, bf16_peak, _, src = _peaks()
    tf = flops / (ms * 1e-3) / 1e12
    chunk_flops = flops - 2.0 * cfg.N * cfg.T * cfg.Dm * cfg.r
    return {"workload": cfg.name, "ms_per_step": ms, "tflops": tf, "flops_per_step": flops,
            "append_ms": append_ms, "chunk_ms": chunk_ms,
            "chunk_tflops": chunk_flops / (chunk_ms * 1e-3) / 1e12,
            "chunk_frac": chunk_flops / (chunk_ms * 1e-3) / 1e12 / bf16_peak,
            "peak_tflops": bf16_peak, "frac": tf / bf16_peak, "peak_source": src,
            "nominal_peak_tflops": NOMINAL_BF16_TFLOPS, "frac_of_nominal": tf / NOMINAL_BF16_TFLOPS,
            "prefill_kernel_traffic": profiled_traffic("prefill_kernel", cfg.name),
            "value_projection": vproj,
            "l2": "256 MB flush before each step"}


def decode_roofline(runner, ms_step):
    """Roofline object of the decode kernel for one timed step of `runner`."""
    hbm, _, _, peak_src = _peaks()
    lb = runner.layer_bytes()
    per_launch_ms = ms_step / runner.launches_per_step
    achieved = lb * len(runner.inp.layers) / (ms_step * 1e-3) / 1e9
    return {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
            "traffic": profiled_traffic("decode_kernel", runner.cfg.name), "peak_source": f"{peak_src} copy bandwidth",
            "nominal_peak": NOMINAL_HBM_GBS, "frac_of_nominal": achieved / NOMINAL_HBM_GBS,
            "kernel": "decode_kernel", "algorithmic_bytes_per_launch": lb,
            "launch_ms": per_launch_ms, "launch_ms_note": "step time / launches per step (gaps included)"}


def time_decode(runner, steps, warmup, sync_all, device_index):
    """Capture the step, then W warm-up and K timed graph replays with the
    clocks sampled throughout; returns (ms per step on this rank, clocks)."""
    import torch.cuda.nvtx as nvtx
    runner.capture()
    clocks = ClockSampler(device_index)
    clocks.start()
    sync_all()
    nvtx.range_push(f"decode {runner.cfg.name}")
    ms = _timed(runner.step, steps, warmup, sync_all)
    nvtx.range_pop()
    return ms / steps, clocks.stop()


def decode_sub_object(cfg, dev, steps, warmup, sync_all, device_index):
    """One more decode workload timed like the headline, as a sub-object of the line."""
    runner = DecodeRunner(cfg, dev)
    ms_step, ck = time_decode(runner, steps, warmup, sync_all, device_index)
    roof = decode_roofline(runner, ms_step)
    out = {"workload": cfg.name, "layers": cfg.layers, "sessions": cfg.S, "agents": cfg.N, "q_heads": cfg.Hq,
           "kv_heads": cfg.Hkv, "rank": cfg.r, "context": cfg.L,
           "mode": "BaseShared" if cfg.mode == 0 else "BaseLRShared", "paged": cfg.paged,
           "ms_per_step": ms_step, "queries_per_s": cfg.queries_per_step / (ms_step * 1e-3),
           "hbm_gbs": roof["achieved"], "frac": roof["frac"], "frac_of_nominal": roof["frac_of_nominal"],
           "algorithmic_bytes_per_launch": roof["algorithmic_bytes_per_launch"], "traffic": roof["traffic"],
           "clocks": ck}
    return out, runner


SWEEP = ("cfg2", "cfg3_1k", "cfg3_2k", "cfg3_4k", "cfg3_8k")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="lrkv", choices=["lrkv", "reference"])
    ap.add_argument("--workload", default="cfg5", choices=[k for k in CONFIGS if k != "cfg4"])
    ap.add_argument("--partition", default="sessions", choices=["sessions", "kv-heads"],
                    help="sessions: every rank runs the whole workload on its own sessions (weak scaling); "
                         "kv-heads: the ranks split one workload's (session, KV head) pairs (strong scaling)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--no-sweep", action="store_true",
                    help="skip the other decode workloads (decode_workloads sub-objects)")
    ap.add_argument("--no-sharing", action="store_true",
                    help="skip the shared / non-shared / full-shared cache comparison")
    ap.add_argument("--layers", type=int, default=None,
                    help="override the layer count (small profiling cases only; not a bench line)")
    ap.add_argument("--context", type=int, default=None,
                    help="override the context length (profiling sweeps only; not a bench line)")
    ap.add_argument("--sessions", type=int, default=None,
                    help="override the session count (profiling sweeps only; not a bench line)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    cfg = CONFIGS[args.workload]
    import dataclasses
    if args.layers is not None:
        cfg = dataclasses.replace(cfg, layers=args.layers)
    if args.context is not None:
        cfg = dataclasses.replace(cfg, L=args.context)
    if args.sessions is not None:
        cfg = dataclasses.replace(cfg, S=args.sessions)

    if args.impl == "reference":
        if rank != 0:
            return
        return run_reference(cfg, args, world)

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

        def sync_all():
            torch.cuda.synchronize()
            dist.barrier()
    else:
        def sync_all():
            torch.cuda.synchronize()

    strong = args.partition == "kv-heads"
    # weak scaling: every rank its own sessions; strong: one workload (one seed), its pairs split over the ranks
    runner = DecodeRunner(cfg, dev, seed_offset=0 if strong else rank_seed_offset(rank))
    if strong:
        runner.set_shard(kv_head_shard_plan(cfg.S, cfg.Hkv, world)[rank])
    ms, ck = time_decode(runner, args.steps, args.warmup, sync_all, local)
    ms_step = max_over_ranks(ms, dev)
    job_queries = cfg.queries_per_step if strong else cfg.queries_per_step * world
    value = job_queries / (ms_step * 1e-3)
    roof = decode_roofline(runner, ms_step)
    lb = roof["algorithmic_bytes_per_launch"]

    e2e = None
    if not args.no_e2e:
        e_ms, hb, db = run_e2e(runner, max(10, args.steps // 10), args.warmup, sync_all)
        e_ms = max_over_ranks(e_ms, dev)
        e2e = {"value": job_queries / (e_ms * 1e-3), "unit": UNIT,
               "h2d_bytes_per_step": hb, "d2h_bytes_per_step": db, "ms_per_step": e_ms}

    # everything below runs on one rank of a one-GPU job only: no collective follows
    single = rank == 0 and world == 1
    cpu = None
    if not args.no_cpu_baseline and single:
        cpu = cpu_baseline_decode(runner)
    launches = runner.launches_per_step * args.steps
    del runner
    torch.cuda.empty_cache()

    prefill = None
    if not args.no_prefill and single:
        prefill = bench_prefill(dev)

    sweep, sharing = None, None
    if single and not (args.no_sweep and args.no_sharing):
        sweep = []
        for key in SWEEP:
            if args.no_sweep and key != "cfg2":
                continue
            sub, r2 = decode_sub_object(CONFIGS[key], dev, args.steps, args.warmup, sync_all, local)
            if not args.no_sweep:
                sweep.append(sub)
            if key == "cfg2" and not args.no_sharing:
                sharing = sharing_comparison(r2)
            del r2
            torch.cuda.empty_cache()
        sweep = sweep or None

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "strong" if strong else "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1) draws of the model shapes)",
            "config": {"workload": cfg.name, "layers": cfg.layers, "sessions": cfg.S, "agents": cfg.N,
                       "q_heads": cfg.Hq, "kv_heads": cfg.Hkv, "head_dim": cfg.d, "rank": cfg.r,
                       "context": cfg.L, "mode": "BaseShared" if cfg.mode == 0 else "BaseLRShared",
                       "paged": cfg.paged, "queries_per_step": cfg.queries_per_step,
                       "parallelism": (f"kv-head shards x{world} (one workload's (session, KV head) pairs split, "
                                       "no collective)") if strong else
                                      f"replicas x{world} (sessions sharded, no collective)",
                       "l2": f"inputs larger than L2: {lb * cfg.layers / 1e9:.2f} GB streamed per step"},
            "hbm_gbs": roof["achieved"],
            "roofline": roof,
            "e2e": e2e,
            "gpu_launches": launches,
            "clocks": ck,
            "cpu_baseline": cpu,
            "decode_workloads": sweep,
            "prefill": prefill,
            "sharing": sharing,
        }
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_reference(cfg, args, world):
    """The oracle as it stands, timed on the host cores, one bounded sample per step."""
    import oracle
    from threadpoolctl import threadpool_info
    from workloads.gen import make_decode_layer, _draw_offsets, seed_for
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed_for(cfg))
    offsets = _draw_offsets(cfg, gen, "cpu")
    import dataclasses
    small = dataclasses.replace(cfg, S=1)
    lay = make_decode_layer(small, gen, "cpu", offsets[:1])
    sl = torch.full((1,), cfg.L, dtype=torch.int32)

    def step():
        oracle.decode(lay.q, lay.k, lay.v, lay.u, lay.b, offsets[:1], sl, cfg.mode, page_table=lay.page_table)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = (time.perf_counter() - t0) / args.steps
    queries = cfg.N / cfg.layers          # one session, one layer of the 28
    value = queries / dt
    cores = len(os.sched_getaffinity(0))
    blas = max([d.get("num_threads", 1) for d in threadpool_info()] + [1])
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded N(0,1) draws of the model shapes)",
        "config": {"workload": cfg.name, "layers": cfg.layers, "sessions": cfg.S, "agents": cfg.N,
                   "context": cfg.L, "parallelism": "host cores"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": min(cores, blas), "kind": "oracle",
                         "sample": f"one session, one layer of {cfg.layers} per step ({cfg.N} agents), fp64 numpy"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))


if __name__ == "__main__":
    main()
