"""Benchmark: STAR-KV latent decode attention on B200.

One step = the whole hot path for one batch: append one new token per sequence
(projection from the hidden state, block Hadamard, 4/3-bit quantize, bit-pack
into the paged cache) and one decode-attention step over the compressed cache
(RoPE'd on-chip key scoring, joint-value contraction, combine, fused output
factors).  Workload: LongChat-7B-shaped layer (32 heads, head_dim 128, hidden
4096), ragged key ranks (mean 32), joint value rank 1024, block Hadamard 32,
4/3-bit latents with fp16 group scales, 16-token pages, batch 16, context 32K.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU (torchrun): each rank runs an independent replica on its own
sequences (the method has no cross-sequence exchange); value = all ranks'
tokens / max-over-ranks time.  Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "latent decode-attn tokens/s & HBM GB/s (% of ~8 TB/s) at ctx 4K-32K, 1 B200"
WORKLOAD = dict(cfg=2, batch=16, ctx=32768, quantized=None)


def workload_spec():
    from synth import gen
    return gen.config_spec(WORKLOAD["cfg"], quantized=WORKLOAD["quantized"])


def workload_label(spec, B, ctx):
    """What the timed step is, in words (shapes of the layer)."""
    if spec.quantized:
        store = (f"block Hadamard {spec.hadamard_block}, " if spec.hadamard_block else "") + \
            f"{spec.top_bits}/{spec.bottom_bits}-bit latents"
    else:
        store = "bf16 latents"
    shape = f"H {spec.n_heads}" + (f"/{spec.n_kv_heads} KV" if spec.n_kv_heads != spec.n_heads else "") + \
        f", d {spec.head_dim}, D {spec.hidden}, R_k {sum(spec.key_ranks)}, r_v {spec.value_rank}, RoPE {spec.rope_theta:g}"
    name = {1: "LongChat-7B-shaped", 2: "LongChat-7B-shaped", 3: "LLaMA-3-8B-shaped GQA"}.get(WORKLOAD["cfg"], "")
    return f"batch {B}, ctx ~{ctx} ({name} layer: {shape}, {store}, 16-token pages)"


def tail_start(ctx, W, K):
    """Tokens cached before the run: W warm-up and K timed steps then append one token each, filling the last
    pages up to ctx."""
    return ctx - 16 * ((W + K + 15) // 16)


def decode_config(spec, B, ctx, W, K, ws, unfused):
    """The `config` of the decode-step line (both arms print the same one)."""
    T0 = tail_start(ctx, W, K)
    return {"workload": "STAR-KV decode step: append 1 token/seq + decode, " + workload_label(spec, B, ctx)
                        + (", unfused value output y_h B_v,h then W_o" if unfused else ""),
            "batch": B, "ctx": ctx, "ctx_range": [T0 + W + 1, T0 + W + K], "parallelism": f"replicas x{ws}",
            "l2": "inputs larger than L2 (the latent cache and M, read once per step)"}


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d.get("hbm_gbs", 6650.0), "measured"
    return 6650.0, "fallback"


def measured_tensor_peak():
    """Dense fp16/bf16 tensor peak in TFLOP/s (the kernels time in a long step: the sustained figure)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d.get("bf16_tflops_sustained", d.get("bf16_tflops", 1400.0)), "measured (sustained bf16)"
    return 1400.0, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    FIELDS = "clocks.sm,clocks.max.sm,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown," \
             "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown," \
             "clocks_event_reasons.sw_power_cap"

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-i", str(self.gpu), "-lms", "100"], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.t.join(timeout=2)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def dist_init():
    import torch
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return rank, ws, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, ws: int) -> float:
    """The maximum of x over the ranks (device times are taken as the slowest rank's)."""
    if ws == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(batch_per_rank: int, ws: int, ms_step_max: float) -> float:
    """Whole-job decode throughput: every rank's sequences over the slowest rank's step time."""
    return batch_per_rank * ws / (ms_step_max * 1e-3)


# ---------------------------------------------------------------------------
# Our arm
# ---------------------------------------------------------------------------

def build_layer(seed_offset: int = 0, unfused: bool = False, max_positions: int = 0):
    """Seeded layer of the workload, loaded into the library."""
    import numpy as np
    import torch
    from decode_attention_rank_b200 import starkv as lib
    from synth import gen
    spec = workload_spec()
    f = gen.make_factors(spec, gen.LAYER_SEED[WORKLOAD["cfg"]])

    def t(x):
        return torch.from_numpy(np.ascontiguousarray(x)).cuda().to(torch.bfloat16)
    A_k = torch.cat([t(a).reshape(-1) for a in f.A_k])
    B_k = torch.cat([t(b).reshape(-1) for b in f.B_k])
    cfg = lib.LayerConfig.from_spec(spec)
    cfg.unfused_output = unfused
    cfg.max_positions = max_positions
    L = lib.load_factors(cfg, A_k, B_k, t(f.A_v), t(f.B_v), t(f.W_o))
    torch.cuda.synchronize()
    return spec, f, L


def fill_cache(spec, f, L, B, T0, rank, ctx, tail_pages):
    """Pool with B sequences of T0 tokens (T0 a multiple of 16), appended in
    latent mode from seeded latents whose columns have the factor spectrum
    (column j ~ N(0, sigma_j^2)).  Two page tables share the filled pages and
    map the tail (positions >= T0) to disjoint zeroed pages, so the timed pass
    and the end-to-end pass each append into fresh slots."""
    import torch
    pages_per_seq = (ctx + 15) // 16
    head = T0 // 16
    n_pages = B * pages_per_seq + B * tail_pages
    g = torch.Generator(device="cuda")
    g.manual_seed(1000 + rank)
    perm = torch.randperm(n_pages, generator=g, device="cuda").to(torch.int32)
    page_table = perm[:B * pages_per_seq].reshape(B, pages_per_seq).contiguous()
    page_table_e2e = page_table.clone()
    page_table_e2e[:, head:head + tail_pages] = perm[B * pages_per_seq:].reshape(B, tail_pages)
    pool = torch.empty(n_pages * L.page_bytes, dtype=torch.uint8, device="cuda")
    L.cache_init(pool, n_pages)
    sig = torch.cat([torch.tensor(s[:r], dtype=torch.float32) for s, r in zip(f.sigma_k, spec.key_ranks)] +
                    [torch.tensor(f.sigma_v[:spec.value_rank], dtype=torch.float32)]).cuda()
    chunk = 4096
    for b in range(B):
        for c0 in range(0, T0, chunk):
            n = min(chunk, T0 - c0)
            z = torch.randn(n, L.latent_total, generator=g, device="cuda") * sig
            seq = torch.full((n,), b, dtype=torch.int32, device="cuda")
            pos = torch.arange(c0, c0 + n, dtype=torch.int32, device="cuda")
            L.append(pool, n_pages, page_table, seq, pos, z, True)
    torch.cuda.synchronize()
    return pool, n_pages, page_table, page_table_e2e


def latent_bytes(spec, r):
    """Algorithmic bytes of one token's latent of rank r (codes + fp16 scales, no page padding)."""
    if not spec.quantized:
        return r * (4 if spec.dtype == "f32" else 2)
    n_hi = math.ceil(spec.top_fraction * r - 1e-9)   # 0.2 * 40 is 8.000000000000002 in floating point
    n_lo = r - n_hi
    bits = spec.top_bits * n_hi + spec.bottom_bits * n_lo
    return bits / 8 + 2 * (math.ceil(n_hi / spec.group_size) + math.ceil(n_lo / spec.group_size))


PHASES = ["query prep + key scoring (k_qprep_tc, k_scores_tc)", "joint value contraction (k_values_tc)",
          "run merge (k_values_combine)", "output through M (k_outproj_tc, k_outproj_reduce)"]


def phase_bytes(spec, B, ctx, unfused=False):
    """Algorithmic HBM bytes of each decode phase: key cache + B'_k; value cache;
    nothing (the merge reads kernel intermediates only); the output factors
    (M, or B'_v per query head and W_o when unfused) + y/out."""
    key = sum(latent_bytes(spec, r) for r in spec.key_ranks)
    val = latent_bytes(spec, spec.value_rank)
    d = spec.head_dim
    out_f = (2 * spec.n_heads * d * (spec.value_rank + spec.hidden) if unfused
             else 2 * spec.n_heads * spec.value_rank * spec.hidden)
    return [B * ctx * key + 2 * d * sum(spec.key_ranks) + B * spec.n_heads * d * 2,
            B * ctx * val,
            0.0,
            out_f + B * spec.hidden * 2]


def phase_flops(spec, B, ctx, unfused=False):
    """Algorithmic tensor flops of each decode phase: 2 r_h d per (token, head) to
    reconstruct, rope and score the keys (the G contraction); 2 r_v per (token,
    query head) for P Z_v; none for the merge; 2 H r_v D per sequence for M
    (unfused: 2 H d (r_v + D))."""
    d = spec.head_dim
    out_f = (B * 2.0 * spec.n_heads * d * (spec.value_rank + spec.hidden) if unfused
             else B * 2.0 * spec.n_heads * spec.value_rank * spec.hidden)
    return [B * ctx * 2.0 * d * sum(spec.key_ranks) * (spec.n_heads // spec.n_kv_heads),
            B * ctx * 2.0 * spec.value_rank * spec.n_heads,
            0.0,
            out_f]


def measured_traffic(phase, tokens):
    """DRAM bytes of one launch of the phase's main kernel, from the ncu capture
    recorded in profiles/dram_traffic.json and scaled by cached tokens; None when
    there is no capture or the kernel's sources changed since it was taken."""
    import hashlib
    try:
        rec = json.load(open(os.path.join(ROOT, "profiles", "dram_traffic.json")))
    except (OSError, ValueError):
        return None
    csrc = os.path.join(ROOT, "decode_attention_rank_b200", "csrc")
    for name, k in rec.get("kernels", {}).items():
        if k.get("phase") != phase:
            continue
        h = hashlib.sha1()
        for f in [k.get("source", name + ".cu"), "tc_common.cuh", "starkv_internal.cuh"]:
            with open(os.path.join(csrc, f), "rb") as fh:
                h.update(fh.read())
        if h.hexdigest() != k.get("source_sha1"):
            return None
        per_launch = k["dram_read_bytes"] + k["dram_write_bytes"]
        # the output GEMM reads the same factors whatever the context length
        return per_launch if not k.get("scales_with_tokens", True) else per_launch * tokens / k["tokens"]
    return None


def decode_bytes(spec, L, B, ctx):
    """Algorithmic HBM bytes of one decode step: cache + B'_k + M + q/out."""
    return B * ctx * L.bytes_per_token + L.factor_bytes + B * (spec.n_heads * spec.head_dim + spec.hidden) * 2


def _oracle_case(T: int):
    """Seeded inputs of one sequence of the workload, and the C++ float64 oracle's decode of it."""
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from harness import Case, queries
    from oracle import cpp as C
    from synth import gen
    c = Case(workload_spec(), gen.LAYER_SEED[WORKLOAD["cfg"]])
    Zs = c.stored(c.latents_direct(0, T))
    q = queries(c, 1)[0, 0]
    B_rot = C.up_projections(c.spec, c.f)
    threads = len(os.sched_getaffinity(0))

    def run():
        C.decode(c.spec, c.f, Zs, q, T - 1, T, B_rot, threads=threads)
    return run, min(threads, c.spec.n_heads)


def cpu_baseline(sample_T: int):
    """Time the float64 C++ oracle on one sequence of the workload (host cores, one thread per head)."""
    run, cores = _oracle_case(sample_T)
    t0 = time.perf_counter()
    run()
    return time.perf_counter() - t0, cores


def run_ours(args, rank, ws, local):
    import torch
    B, ctx = WORKLOAD["batch"], WORKLOAD["ctx"]
    K, W = args.steps, args.warmup
    spec, f, L = build_layer(unfused=args.unfused)
    tail_pages = (W + K + 15) // 16
    T0 = tail_start(ctx, W, K)      # each step appends one token at T0 + i and decodes T0 + i + 1 tokens
    pool, n_pages, page_table, page_table_e2e = fill_cache(spec, f, L, B, T0, rank, ctx, tail_pages)
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream()
    g = torch.Generator(device="cuda")
    g.manual_seed(77 + rank)
    x_all = torch.randn(W + K, B, spec.hidden, generator=g, device=dev).to(torch.bfloat16)
    q_all = (torch.randn(W + K, B, spec.n_heads, spec.head_dim, generator=g, device=dev) /
             math.sqrt(spec.head_dim)).to(torch.bfloat16)
    out = torch.empty(B, spec.hidden, dtype=torch.bfloat16, device=dev)
    ws_dec = torch.empty(L.workspace_bytes(B, page_table.shape[1] * 16), dtype=torch.uint8, device=dev)
    ws_app = torch.empty(max(L.append_workspace_bytes(B), 256), dtype=torch.uint8, device=dev)
    seq_idx = torch.arange(B, dtype=torch.int32, device=dev)
    lens = (torch.arange(W + K, dtype=torch.int32, device=dev)[:, None] + (T0 + 1)).repeat(1, B).contiguous()
    pos_all = (lens - 1).contiguous()

    def step(i, pt, ev=None):
        L.append(pool, n_pages, pt, seq_idx, pos_all[i], x_all[i], False, workspace=ws_app)
        if ev is not None:
            ev[0].record(stream)
        L.decode(pool, n_pages, pt, lens[i], q_all[i], out, ws_dec)
        if ev is not None:
            ev[1].record(stream)

    for i in range(W):
        step(i, page_table)
    torch.cuda.synchronize()
    barrier(ws)
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    barrier(ws)
    L.profile_decode(K)   # CUDA events between the decode's kernels, on its stream
    torch.cuda.nvtx.range_push("timed")
    t_start.record(stream)
    for k in range(K):
        step(W + k, page_table, evs[k])
    t_end.record(stream)
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    barrier(ws)
    ms_total = t_start.elapsed_time(t_end)
    dec_ms = sum(a.elapsed_time(b) for a, b in evs) / K
    ph = L.decode_phase_ms(K)
    L.profile_decode(0)
    ph_ms = [max_over_ranks(sum(c[p] for c in ph) / K, ws) for p in range(len(PHASES))]
    clk = clocks.stop()
    assert L.sync_status() == 0, "device status word set during the benchmark"
    ms_step = max_over_ranks(ms_total / K, ws)
    dec_ms = max_over_ranks(dec_ms, ws)

    # End to end through the C ABI with host buffers: every step copies its inputs
    # (x, q, lengths, positions) from pinned host memory and reads the output back.
    pin_x = x_all.cpu().pin_memory()
    pin_q = q_all.cpu().pin_memory()
    pin_len = lens.cpu().pin_memory()
    pin_pos = pos_all.cpu().pin_memory()
    pin_out = torch.empty(W + K, B, spec.hidden, dtype=torch.bfloat16).pin_memory()
    x_d, q_d = torch.empty_like(x_all[0]), torch.empty_like(q_all[0])
    len_d, pos_d = torch.empty_like(lens[0]), torch.empty_like(lens[0])

    def e2e_step(i):
        x_d.copy_(pin_x[i], non_blocking=True)
        q_d.copy_(pin_q[i], non_blocking=True)
        len_d.copy_(pin_len[i], non_blocking=True)
        pos_d.copy_(pin_pos[i], non_blocking=True)
        L.append(pool, n_pages, page_table_e2e, seq_idx, pos_d, x_d, False, workspace=ws_app)
        L.decode(pool, n_pages, page_table_e2e, len_d, q_d, out, ws_dec)
        pin_out[i].copy_(out, non_blocking=True)

    for i in range(W):
        e2e_step(i)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    barrier(ws)
    e0.record(stream)
    for k in range(K):
        e2e_step(W + k)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / K, ws)
    h2d = (x_d.numel() + q_d.numel()) * 2 + (len_d.numel() + pos_d.numel()) * 4
    d2h = out.numel() * 2

    peak, peak_kind = measured_peaks()
    dbytes = decode_bytes(spec, L, B, T0 + W + K // 2)
    achieved = dbytes / (dec_ms * 1e-3) / 1e9
    pbytes = phase_bytes(spec, B, T0 + W + K // 2, args.unfused)
    pflops = phase_flops(spec, B, T0 + W + K // 2, args.unfused)
    tpeak, tpeak_kind = measured_tensor_peak()
    kernels = [{"phase": PHASES[p], "us": ph_ms[p] * 1e3, "algorithmic_bytes": pbytes[p],
                "GB/s": (pbytes[p] / (ph_ms[p] * 1e-3) / 1e9) if ph_ms[p] > 0 else None,
                "frac": (pbytes[p] / (ph_ms[p] * 1e-3) / 1e9 / peak) if ph_ms[p] > 0 else None,
                # tensor-pipe co-bound: algorithmic flops over the measured dense fp16 peak
                "algorithmic_flops": pflops[p],
                "TFLOP/s": (pflops[p] / (ph_ms[p] * 1e-3) / 1e12) if ph_ms[p] > 0 else None,
                "tensor_frac": (pflops[p] / (ph_ms[p] * 1e-3) / 1e12 / tpeak) if ph_ms[p] > 0 else None}
               for p in range(len(PHASES))]
    dom = max(range(len(PHASES)), key=lambda p: ph_ms[p])
    tokens_per_s = job_tokens_per_s(B, ws, ms_step)
    res = {
        "metric": METRIC,
        "value": tokens_per_s,
        "unit": "tokens/s",
        "n_gpus": ws,
        "steps": K,
        "warmup": W,
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": ("u3/u4 latent codes + fp16 scales, bf16 factors/q/out, fp32 accumulate" if spec.quantized
                  else "bf16 latents/factors/q/out, fp32 accumulate"),
        "data": "synthetic (seeded latents with the factor spectrum; random-init factors)",
        "config": decode_config(spec, B, ctx, W, K, ws, args.unfused),
        "input_bytes": {"latent_cache": B * ctx * L.bytes_per_token, "factors": L.factor_bytes, "l2": 126 << 20},
        "us_per_layer_step": ms_step * 1e3,
        "decode_us": dec_ms * 1e3,
        "roofline": {"bound": "hbm", "kernel": PHASES[dom], "achieved": kernels[dom]["GB/s"], "peak": peak,
                     "peak_kind": peak_kind, "unit": "GB/s", "frac": kernels[dom]["frac"],
                     "traffic": measured_traffic(dom, B * (T0 + W + K // 2)),
                     "algorithmic_bytes": pbytes[dom], "us_per_launch": ph_ms[dom] * 1e3,
                     "whole_decode": {"achieved": achieved, "frac": achieved / peak, "algorithmic_bytes": dbytes,
                                      "us": dec_ms * 1e3},
                     "tensor_cobound": {"achieved": kernels[dom]["TFLOP/s"], "peak": tpeak, "peak_kind": tpeak_kind,
                                        "unit": "TFLOP/s", "frac": kernels[dom]["tensor_frac"],
                                        "algorithmic_flops": pflops[dom]}},
        "kernels": kernels,
        "e2e": {"value": B * ws / (e2e_ms * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        # append: 4 kernels; decode: 6 (unfused output: 9); see the launch list under profiles/
        "gpu_launches": K * (13 if args.unfused else 10),
        "clocks": clk,
    }
    if args.unfused:
        res["mode"] = "unfused value output"
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        dt, cores = cpu_baseline(ctx)
        res["cpu_baseline"] = {"value": 1.0 / dt, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                               "sample": f"1 sequence of the batch at ctx {ctx}: float64 C++ oracle, explicit K/V "
                                         f"reconstruction + softmax attention + W_o ({dt:.1f} s)"}
    return res


def run_reference(args, rank, ws):
    """The oracle, as it stands, on the host cores: one sequence of the workload per step, reported on the
    decode step's own config."""
    if rank != 0:
        return None
    B, ctx = WORKLOAD["batch"], WORKLOAD["ctx"]
    K, W = args.steps, args.warmup
    T = args.ref_ctx or ctx
    run, cores = _oracle_case(T)
    for _ in range(W):
        run()
    t0 = time.perf_counter()
    for _ in range(K):
        run()
    dt = (time.perf_counter() - t0) / K
    v = 1.0 / dt
    return {"metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": ws, "steps": K, "warmup": W,
            "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": decode_config(workload_spec(), B, ctx, W, K, ws, args.unfused),
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": f"1 of the {B} sequences per step, decoded at ctx {T} by the float64 C++ "
                                       "oracle (explicit K/V reconstruction + softmax attention + W_o)"},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def run_prefill(args):
    """Time one causal prefill chunk: `args.prefill` queries after ctx - prefill
    tokens of history, batch 1, on the workload's layer (separate JSON line;
    not the headline metric)."""
    import torch
    n = args.prefill
    T = WORKLOAD["ctx"] if args.ctx else 4096
    assert T % 16 == 0 and 0 < n <= T, "prefill chunk must fit the context"
    torch.cuda.set_device(0)
    spec, f, L = build_layer()
    pool, n_pages, page_table, _ = fill_cache(spec, f, L, 1, T, 0, T, 0)
    g = torch.Generator(device="cuda")
    g.manual_seed(91)
    q = (torch.randn(n, spec.n_heads, spec.head_dim, generator=g, device="cuda") /
         math.sqrt(spec.head_dim)).to(torch.bfloat16)
    out = torch.empty(n, spec.hidden, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(L.workspace_bytes(1, T, n), dtype=torch.uint8, device="cuda")
    for _ in range(args.warmup):
        L.prefill(pool, n_pages, page_table, [T - n], [n], q, out, ws)
    torch.cuda.synchronize()
    clocks = ClockSampler(0)
    clocks.start()
    time.sleep(0.3)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.nvtx.range_push("timed")
    e0.record()
    for _ in range(args.steps):
        L.prefill(pool, n_pages, page_table, [T - n], [n], q, out, ws)
    e1.record()
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    clk = clocks.stop()
    status = L.sync_status()
    ms = e0.elapsed_time(e1) / args.steps
    # algorithmic tensor flops of the chunk: S = QK^T and O += PV over the visible (query, key) pairs of every
    # head, the key and value rebuild of the T cached tokens, and the output through W_o
    d, H, Hkv = spec.head_dim, spec.n_heads, spec.n_kv_heads
    pairs = n * (T - n) + n * (n + 1) // 2
    flops = (4.0 * d * pairs * H + 2.0 * T * d * sum(spec.key_ranks) + 2.0 * T * spec.value_rank * Hkv * d +
             2.0 * n * H * d * spec.hidden)
    tpk, tsrc = measured_tensor_peak()
    ach = flops / (ms * 1e-3) / 1e12
    return {"metric": "causal prefill query tokens/s (latent attention over the paged cache)", "value": n / (ms * 1e-3),
            "unit": "query tokens/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "u3/u4 latent codes + fp16 "
            "scales, bf16 factors/q/out, fp32 accumulate", "data": "synthetic", "mode": "prefill",
            "config": {"workload": f"prefill chunk of {n} queries after {T - n} tokens of history, batch 1 "
                                   "(LongChat-7B-shaped layer, 4/3-bit latents)", "batch": 1, "ctx": T,
                       "queries": n},
            "roofline": {"bound": "tensor", "achieved": ach, "peak": tpk, "unit": "TFLOP/s", "frac": ach / tpk,
                         "traffic": None, "peak_source": tsrc, "algorithmic_flops": flops},
            "clocks": clk, "device_status": status}


def run_plain(args):
    """Time the decode of one uncompressed (plain) layer of the 32-layer stack
    (K stored after RoPE and V in bf16 pages; the streaming split-K kernel
    k_plain_decode, the run merge and the tensor-core output GEMM): batch and ctx from --batch/--ctx (default 16
    and 4096).  Separate JSON line; not the headline metric."""
    import numpy as np
    import torch
    from decode_attention_rank_b200 import starkv as lib
    from synth import gen
    B = args.batch or 16
    T = args.ctx or 4096
    assert T % 16 == 0
    torch.cuda.set_device(0)
    spec = gen.config_spec(4, layer=0)
    f = gen.make_factors(spec, gen.LAYER_SEED[4], 0)

    def t(x):
        return torch.from_numpy(np.ascontiguousarray(x)).cuda().to(torch.bfloat16)
    L = lib.load_factors(lib.LayerConfig.from_spec(spec), t(f.W_k), None, t(f.W_v), None, t(f.W_o))
    pages = T // 16 + 1
    n_pages = B * pages
    g = torch.Generator(device="cuda")
    g.manual_seed(2024)
    page_table = torch.randperm(n_pages, generator=g, device="cuda").to(torch.int32).reshape(B, pages).contiguous()
    pool = torch.empty(n_pages * L.page_bytes, dtype=torch.uint8, device="cuda")
    L.cache_init(pool, n_pages)
    for b in range(B):
        for c0 in range(0, T, 4096):
            n = min(4096, T - c0)
            z = torch.randn(n, L.latent_total, generator=g, device="cuda")
            L.append(pool, n_pages, page_table, torch.full((n,), b, dtype=torch.int32, device="cuda"),
                     torch.arange(c0, c0 + n, dtype=torch.int32, device="cuda"), z, True)
    q = (torch.randn(B, spec.n_heads, spec.head_dim, generator=g, device="cuda") /
         math.sqrt(spec.head_dim)).to(torch.bfloat16)
    out = torch.empty(B, spec.hidden, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(L.workspace_bytes(B, pages * 16), dtype=torch.uint8, device="cuda")
    lens = torch.full((B,), T, dtype=torch.int32, device="cuda")
    clocks = ClockSampler(0)
    clocks.start()
    time.sleep(0.3)
    ms = _time_decodes(L, pool, n_pages, page_table, lens, q, out, ws, args.steps, args.warmup)
    clk = clocks.stop()
    status = L.sync_status()
    peak, peak_kind = measured_peaks()
    # algorithmic bytes: K and V of every cached token (bf16) + W_o + q/out
    dbytes = B * T * 2 * 2 * spec.n_kv_heads * spec.head_dim + 2 * spec.n_heads * spec.head_dim * spec.hidden + \
        B * (spec.n_heads * spec.head_dim + spec.hidden) * 2
    gbs = dbytes / (ms * 1e-3) / 1e9
    return {"metric": "plain-layer decode tokens/s (uncompressed bf16 K/V)", "value": B / (ms * 1e-3),
            "unit": "tokens/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16 K/V, fp32 accumulate",
            "data": "synthetic", "mode": "plain",
            "config": {"workload": f"plain layer (workload-4 layers 0, 1, 31) decode, batch {B}, ctx {T}",
                       "batch": B, "ctx": T},
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                         "frac": gbs / peak, "algorithmic_bytes": dbytes},
            "clocks": clk, "device_status": status}


def _time_decodes(L, pool, n_pages, page_table, lens, q, out, ws, steps, warmup):
    import torch
    for _ in range(warmup):
        L.decode(pool, n_pages, page_table, lens, q, out, ws)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.nvtx.range_push("timed")
    e0.record()
    for _ in range(steps):
        L.decode(pool, n_pages, page_table, lens, q, out, ws)
    e1.record()
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    assert L.sync_status() == 0
    return e0.elapsed_time(e1) / steps


def run_compare_plain(args):
    """The in-house counterpart of the reading notes' attention-module speed-up
    (section 8.1-8.2: latent attention against uncompressed attention at batch
    16, long contexts): decode of one uncompressed bf16 layer (plain K/V) and of
    one 4/3-bit latent layer of the same LongChat-7B / LLaMA-2-7B shape (H 32,
    d 128, D 4096) at batch 16 over a list of contexts, one JSON line."""
    import numpy as np
    import torch
    from decode_attention_rank_b200 import starkv as lib
    from synth import gen
    torch.cuda.set_device(0)
    B = args.batch or 16
    ctxs = [int(x) for x in args.compare_plain.split(",")]
    pspec = gen.config_spec(4, layer=0)
    pf = gen.make_factors(pspec, gen.LAYER_SEED[4], 0)

    def t(x):
        return torch.from_numpy(np.ascontiguousarray(x)).cuda().to(torch.bfloat16)
    pcfg = lib.LayerConfig.from_spec(pspec)
    PL = lib.load_factors(pcfg, t(pf.W_k), None, t(pf.W_v), None, t(pf.W_o))
    clocks = ClockSampler(0)
    clocks.start()
    rows = []
    g = torch.Generator(device="cuda")
    g.manual_seed(4242)
    q = (torch.randn(B, 32, 128, generator=g, device="cuda") / math.sqrt(128)).to(torch.bfloat16)
    out = torch.empty(B, 4096, dtype=torch.bfloat16, device="cuda")
    for T in ctxs:
        pages = T // 16
        lens = torch.full((B,), T, dtype=torch.int32, device="cuda")
        # plain layer: K (after RoPE) and V, bf16
        n_pages = B * pages
        pt = torch.randperm(n_pages, generator=g, device="cuda").to(torch.int32).reshape(B, pages).contiguous()
        pool = torch.empty(n_pages * PL.page_bytes, dtype=torch.uint8, device="cuda")
        PL.cache_init(pool, n_pages)
        for b in range(B):
            for c0 in range(0, T, 4096):
                n = min(4096, T - c0)
                z = torch.randn(n, PL.latent_total, generator=g, device="cuda")
                PL.append(pool, n_pages, pt, torch.full((n,), b, dtype=torch.int32, device="cuda"),
                          torch.arange(c0, c0 + n, dtype=torch.int32, device="cuda"), z, True)
        ws = torch.empty(PL.workspace_bytes(B, pages * 16), dtype=torch.uint8, device="cuda")
        ms_plain = _time_decodes(PL, pool, n_pages, pt, lens, q, out, ws, args.steps, args.warmup)
        plain_bytes = B * T * PL.bytes_per_token + PL.factor_bytes
        del pool, ws
        torch.cuda.empty_cache()
        # latent layer (4/3-bit, block Hadamard), RoPE table covering the context
        spec, f, L = build_layer(max_positions=max(T, 32768))
        lpool, ln_pages, lpt, _ = fill_cache(spec, f, L, B, T, 0, T, 0)
        lws = torch.empty(L.workspace_bytes(B, lpt.shape[1] * 16), dtype=torch.uint8, device="cuda")
        ms_lat = _time_decodes(L, lpool, ln_pages, lpt, lens, q, out, lws, args.steps, args.warmup)
        lat_bytes = B * T * L.bytes_per_token + L.factor_bytes
        del lpool, lws, L
        torch.cuda.empty_cache()
        rows.append({"ctx": T, "plain_us": ms_plain * 1e3, "latent_us": ms_lat * 1e3,
                     "speedup": ms_plain / ms_lat,
                     "plain_GBps": plain_bytes / (ms_plain * 1e-3) / 1e9,
                     "latent_GBps": lat_bytes / (ms_lat * 1e-3) / 1e9,
                     "plain_bytes": plain_bytes, "latent_bytes": lat_bytes})
    clk = clocks.stop()
    peak, peak_kind = measured_peaks()
    return {"metric": "attention-module decode speed-up, latent 4/3-bit layer vs uncompressed bf16 layer",
            "value": rows[-1]["speedup"], "unit": "x (plain time / latent time)", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16 K/V vs u3/u4 latent codes + fp16 scales", "data": "synthetic",
            "mode": "compare_plain",
            "config": {"workload": f"decode of one LongChat-7B / LLaMA-2-7B-shaped attention layer (H 32, d 128, "
                                   f"D 4096), batch {B}: uncompressed bf16 K/V against STAR-KV 4/3-bit latents "
                                   f"(ragged key ranks mean 32, r_v 1024, fused M_h)", "batch": B, "ctxs": ctxs},
            "points": rows, "hbm_peak": peak, "hbm_peak_kind": peak_kind, "clocks": clk}


def _stack_layer(layer: int, max_positions: int):
    """Layer `layer` of the 32-layer LongChat-7B-shaped stack: layers 0, 1 and 31 uncompressed (bf16 K/V),
    the others 4/3-bit latents with block Hadamard and their own seeded ragged key ranks.  For timing only
    the factors are seeded random bf16 tensors of the right shapes (the cost does not depend on their
    values; parity is tested with the SVD factors elsewhere)."""
    import torch
    from decode_attention_rank_b200 import starkv as lib
    from synth import gen
    spec = gen.config_spec(4, layer=layer)
    g = torch.Generator(device="cuda")
    g.manual_seed(7000 + layer)
    D, d, H, Hkv = spec.hidden, spec.head_dim, spec.n_heads, spec.n_kv_heads

    def r(*shape, scale=1.0):
        return (torch.randn(*shape, generator=g, device="cuda") * scale).to(torch.bfloat16)
    cfg = lib.LayerConfig.from_spec(spec)
    cfg.max_positions = max_positions
    if spec.plain:
        return spec, lib.load_factors(cfg, r(D, Hkv * d, scale=D ** -0.5), None, r(D, Hkv * d, scale=D ** -0.5),
                                      None, r(H * d, D, scale=D ** -0.5))
    Rk = sum(spec.key_ranks)
    return spec, lib.load_factors(cfg, r(D * Rk, scale=D ** -0.5), r(Rk * d, scale=d ** -0.5),
                                  r(D, spec.value_rank, scale=D ** -0.5), r(spec.value_rank, Hkv * d, scale=0.03),
                                  r(H * d, D, scale=D ** -0.5))


def _fill_random(L, B, T, g):
    """Page table and pool of B sequences of T tokens, appended in latent mode from seeded normals."""
    import torch
    pages = (T + 15) // 16
    n_pages = B * pages
    pt = torch.randperm(n_pages, generator=g, device="cuda").to(torch.int32).reshape(B, pages).contiguous()
    pool = torch.empty(n_pages * L.page_bytes, dtype=torch.uint8, device="cuda")
    L.cache_init(pool, n_pages)
    chunk = max(16, min(T, (1 << 26) // max(1, L.latent_total * 4)) // 16 * 16)
    for b in range(B):
        for c0 in range(0, T, chunk):
            n = min(chunk, T - c0)
            z = torch.randn(n, L.latent_total, generator=g, device="cuda") * 0.3
            L.append(pool, n_pages, pt, torch.full((n,), b, dtype=torch.int32, device="cuda"),
                     torch.arange(c0, c0 + n, dtype=torch.int32, device="cuda"), z, True)
    return pool, n_pages, pt


def run_stack(args):
    """The 32-layer stack of the long-context workload: a causal chunked prefill of 4096 tokens (chunks of
    1024, each appended before its attention) and a decode-step sweep over batch x context, the step time
    being the sum over the 32 layers.  The layers are timed one at a time (each with its own cache, built,
    timed and freed), since the whole stack's caches at batch 64 and 32K tokens (~175 GB) would not fit
    beside the workspaces.  One JSON line."""
    import torch
    torch.cuda.set_device(0)
    points = [tuple(int(x) for x in p.split("x")) for p in args.stack.split(",")]
    g = torch.Generator(device="cuda")
    g.manual_seed(31337)
    clocks = ClockSampler(0)
    clocks.start()
    # prefill: batch 1, 4096 tokens in four chunks of 1024
    pre_ms = [0.0] * 32
    n_chunk, T_pre = 1024, 4096
    for layer in range(32):
        spec, L = _stack_layer(layer, 32768)
        pages = T_pre // 16
        pt = torch.randperm(pages, generator=g, device="cuda").to(torch.int32).reshape(1, pages).contiguous()
        pool = torch.empty(pages * L.page_bytes, dtype=torch.uint8, device="cuda")
        L.cache_init(pool, pages)
        x = (torch.randn(T_pre, spec.hidden, generator=g, device="cuda")).to(torch.bfloat16)
        q = (torch.randn(T_pre, spec.n_heads, spec.head_dim, generator=g, device="cuda") /
             math.sqrt(spec.head_dim)).to(torch.bfloat16)
        out = torch.empty(n_chunk, spec.hidden, dtype=torch.bfloat16, device="cuda")
        ws = torch.empty(L.workspace_bytes(1, T_pre, n_chunk), dtype=torch.uint8, device="cuda")
        wsa = torch.empty(max(256, L.append_workspace_bytes(n_chunk)), dtype=torch.uint8, device="cuda")
        seq = torch.zeros(n_chunk, dtype=torch.int32, device="cuda")
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for c in range(T_pre // n_chunk):
            pos = torch.arange(c * n_chunk, (c + 1) * n_chunk, dtype=torch.int32, device="cuda")
            L.append(pool, pages, pt, seq, pos, x[c * n_chunk:(c + 1) * n_chunk], False, workspace=wsa)
            L.prefill(pool, pages, pt, [c * n_chunk], [n_chunk], q[c * n_chunk:(c + 1) * n_chunk], out, ws)
        e1.record()
        torch.cuda.synchronize()
        assert L.sync_status() == 0
        pre_ms[layer] = e0.elapsed_time(e1)
        del pool, ws, wsa, L
        torch.cuda.empty_cache()
    # decode sweep
    sweep = []
    for B, T in points:
        per_layer = [0.0] * 32
        for layer in range(32):
            spec, L = _stack_layer(layer, max(T, 32768))
            pool, n_pages, pt = _fill_random(L, B, T, g)
            q = (torch.randn(B, spec.n_heads, spec.head_dim, generator=g, device="cuda") /
                 math.sqrt(spec.head_dim)).to(torch.bfloat16)
            out = torch.empty(B, spec.hidden, dtype=torch.bfloat16, device="cuda")
            ws = torch.empty(L.workspace_bytes(B, pt.shape[1] * 16), dtype=torch.uint8, device="cuda")
            lens = torch.full((B,), T, dtype=torch.int32, device="cuda")
            per_layer[layer] = _time_decodes(L, pool, n_pages, pt, lens, q, out, ws, args.steps, args.warmup)
            del pool, ws, L
            torch.cuda.empty_cache()
        step_ms = sum(per_layer)
        sweep.append({"batch": B, "ctx": T, "step_ms": step_ms, "tokens_per_s": B / (step_ms * 1e-3),
                      "plain_layer_ms": [per_layer[i] for i in (0, 1, 31)],
                      "compressed_layer_ms_mean": sum(per_layer[2:31]) / 29,
                      "compressed_layer_ms_min_max": [min(per_layer[2:31]), max(per_layer[2:31])]})
    clk = clocks.stop()
    return {"metric": "32-layer stack: chunked prefill time and decode tokens/s over batch x context", "mode": "stack",
            "value": sweep[-1]["tokens_per_s"] if sweep else None, "unit": "tokens/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "u3/u4 latent codes + fp16 scales (layers 2-30), bf16 K/V (0, 1, 31)",
            "data": "synthetic (seeded random factors and latents; layers timed one at a time)",
            "config": {"workload": "LongChat-7B-shaped 32-layer stack (attention only): layers 0, 1, 31 uncompressed, "
                                   "2-30 4/3-bit latents with block Hadamard and per-layer ragged key ranks; prefill "
                                   "4096 tokens in chunks of 1024, batch 1; decode sweep", "points": points},
            "prefill": {"tokens": T_pre, "chunk": n_chunk, "total_ms": sum(pre_ms),
                        "plain_layer_ms": [pre_ms[i] for i in (0, 1, 31)],
                        "compressed_layer_ms_mean": sum(pre_ms[2:31]) / 29,
                        "tokens_per_s": T_pre / (sum(pre_ms) * 1e-3)},
            "sweep": sweep, "clocks": clk}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ref-ctx", type=int, default=0)
    ap.add_argument("--ctx", type=int, default=0, help="context length (default: the headline 32768); a smaller "
                    "value gives the small case used for profiler captures")
    ap.add_argument("--batch", type=int, default=0, help="sequences per step (default 16)")
    ap.add_argument("--prefill", type=int, default=0, help="time a causal prefill chunk of this many queries "
                    "(history = ctx - queries, ctx default 4096) instead of the decode step")
    ap.add_argument("--cfg", type=int, default=0, help="time the decode step of workload 1, 2 or 3 at its own "
                    "batch and context (default: workload 2, the headline)")
    ap.add_argument("--quantized", action="store_true", help="with --cfg 3: the 4/3-bit variant")
    ap.add_argument("--unfused", action="store_true", help="the workload with the unfused value output "
                    "(y_h B_v,h then W_o) instead of the fused M_h (separate line; the fused form is the headline)")
    ap.add_argument("--plain", action="store_true", help="time the decode of an uncompressed layer of the "
                    "32-layer stack instead (batch/ctx from --batch/--ctx, default 16 and 4096)")
    ap.add_argument("--compare-plain", default="", help="comma-separated contexts: time an uncompressed layer "
                    "against a 4/3-bit latent layer at each (batch from --batch, default 16); one JSON line")
    ap.add_argument("--stack", default="", help="comma-separated BxT decode points for the 32-layer stack "
                    "(e.g. 1x4096,16x32768); also times its 4096-token chunked prefill; one JSON line")
    args = ap.parse_args()
    if args.stack:
        print(json.dumps(run_stack(args)), flush=True)
        return
    if args.compare_plain:
        print(json.dumps(run_compare_plain(args)), flush=True)
        return
    if args.plain:
        print(json.dumps(run_plain(args)), flush=True)
        return
    if args.cfg:
        from synth import gen
        assert args.cfg in (1, 2, 3), "--cfg takes 1, 2 or 3"
        WORKLOAD["cfg"] = args.cfg
        WORKLOAD["batch"] = gen.CONFIG_SHAPES[args.cfg]["batch"]
        WORKLOAD["ctx"] = gen.CONFIG_SHAPES[args.cfg]["ctx"]
        WORKLOAD["quantized"] = bool(args.quantized) if args.cfg == 3 else None
    if args.ctx:
        WORKLOAD["ctx"] = args.ctx
    if args.batch:
        WORKLOAD["batch"] = args.batch
    if args.prefill:
        print(json.dumps(run_prefill(args)), flush=True)
        return
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        ws = int(os.environ.get("WORLD_SIZE", "1"))
        res = run_reference(args, rank, ws)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    rank, ws, local = dist_init()
    res = run_ours(args, rank, ws, local)
    if rank == 0:
        print(json.dumps(res), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
