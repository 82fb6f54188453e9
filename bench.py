"""Benchmark of the paged KV cache hot path on B200.

One step = kv_append of every new token (norm, RoPE, 16-bit conversion,
scatter) followed by paged_decode_attention over every decoding sequence
(and, for a mixed workload, paged_prefill_attention over the prefill
chunks), by default on the Llama-3-8B-shaped batch-32 decode workload
(Hq=32, Hkv=8, D=128, bf16 pool, block size 16, contexts U[512, 4096]).
Inputs are synthetic and seeded.

Reports whole-step KV-read throughput (algorithmic K+V bytes of the decode
pass divided by the step time), the decode kernel against the measured HBM
roofline, an end-to-end figure through the C ABI with host buffers, the CPU
oracle timed on this host, and the SM clocks seen during the timed region.

Usage:  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
        under torchrun for N > 1 (one rank per GPU, independent replicas).
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "paged decode attn KV-read GB/s (% of HBM peak); seq-steps/s at batch 32"
WORKLOAD = "llama3-8b-b32"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
DECODE_SOURCES = ("paged_kv_cache_321_b200/csrc/decode.cu", "paged_kv_cache_321_b200/csrc/common.cuh")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=WORKLOAD)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--split-tokens", type=int, default=0)
    return ap.parse_args()


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def measured_bf16_tflops():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"]), "measured burst"
    except Exception:
        return 1590.0, "fallback"


def sources_sha(paths) -> str:
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def decode_kernel_name(sp) -> str:
    """The decode kernel the library picks for this shape (tensor-core tile
    products for groups of 4 and 8 with blocks of at least 16 tokens)."""
    G = sp.Hq // sp.Hkv
    if G in (4, 8) and sp.bs >= 16 and sp.D % 64 == 0:
        return "kvp::dec::decode_tc_kernel (+ merge grid)"
    return "kvp::dec::decode_kernel"


def ncu_traffic(workload: str):
    """DRAM bytes per decode launch from the committed ncu summary, or None
    when the kernel sources changed since that capture."""
    path = os.path.join(ROOT, "profiles", f"decode_{workload}.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except Exception:
        return None
    if d.get("sources_sha") != sources_sha(DECODE_SOURCES):
        return None
    return d.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        time.sleep(0.1)
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        sm, mx, reasons = [], None, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup(n_gpus: int):
    import torch

    from paged_kv_cache_321_b200 import replicas

    rank, world, local = replicas.world_from_env()
    if n_gpus <= 1 or world == 1:
        return 0, 1, None
    torch.cuda.set_device(local)
    dist = replicas.init("nccl", timeout_s=120, device=torch.device("cuda", local))
    return rank, world, dist


# ------------------------------------------------------------------ oracle
def oracle_step(orc, wl, seqs, threads):
    """The oracle's step restricted to the given sequences: their new tokens'
    append, then their decode attention."""
    sp = wl.spec
    tok = wl.cu_q[seqs]
    pk = wl.pool_k[sp.layer].copy()
    pv = wl.pool_v[sp.layer].copy()
    rope = orc.rope_table(float(np.float32(sp.theta)), sp.D, wl.max_seq_len, sp.rope_dim) if sp.theta else None
    st, q_out = orc.kv_append(Hq=sp.Hq, Hkv=sp.Hkv, D=sp.D, bs=sp.bs, kv_dtype=sp.kv_dtype, q=wl.q[tok], k=wl.k[tok],
                              v=wl.v[tok], tok_req=wl.tok_req[tok], positions=wl.positions[tok],
                              block_tables=wl.block_tables, pool_k=pk, pool_v=pv, max_seq_len=wl.max_seq_len,
                              q_norm_w=wl.q_norm_w, k_norm_w=wl.k_norm_w, eps=sp.eps, rope=rope,
                              rope_dim=sp.rope_dim, rope_style=sp.rope_style, window=sp.window)
    st2, out, _ = orc.paged_attention(Hq=sp.Hq, Hkv=sp.Hkv, D=sp.D, bs=sp.bs, kv_dtype=sp.kv_dtype,
                                      q=q_out.reshape(-1, sp.Hq, sp.D), q_seq=seqs, q_pos=wl.ctx[seqs] - 1,
                                      block_tables=wl.block_tables, pool_k=pk, pool_v=pv, threads=threads,
                                      window=sp.window)
    return st | st2


def cpu_baseline(wl, budget_s=12.0, threads=None):
    import oracle as orc

    threads = threads or os.cpu_count() or 1
    seqs = wl.decode_seqs
    t0 = time.perf_counter()
    reps, nbytes = 0, 0
    while True:
        oracle_step(orc, wl, seqs, threads)
        reps += 1
        nbytes += wl.kv_read_bytes(seqs)
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    return {"value": round(nbytes / dt / 1e9, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
            "sample": f"{reps} full step(s) of {wl.spec.name}: append of {len(seqs)} tokens + fp64 attention over "
                      f"{len(seqs)} sequences ({wl.kv_read_bytes(seqs) / 1e6:.1f} MB KV each)",
            "seconds": round(dt, 2)}


def run_reference(args):
    """The reference arm: the CPU oracle, as it stands, on this host."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle as orc
    from workloads import SPECS, make_workload

    wl = make_workload(SPECS[args.workload])
    threads = os.cpu_count() or 1
    seqs_all = wl.decode_seqs
    # size one step so the whole run stays within about two minutes
    t0 = time.perf_counter()
    oracle_step(orc, wl, seqs_all[:1], threads)
    one = time.perf_counter() - t0
    total = args.steps + args.warmup
    n = int(max(1, min(len(seqs_all), 120.0 / max(total * one, 1e-9))))
    seqs = seqs_all[:n]
    for _ in range(args.warmup):
        oracle_step(orc, wl, seqs, threads)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(orc, wl, seqs, threads)
    dt = time.perf_counter() - t0
    gbs = wl.kv_read_bytes(seqs) * args.steps / dt / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": round(gbs, 4), "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload, "sample_sequences": n, "of_sequences": len(seqs_all)},
        "cpu_baseline": {"value": round(gbs, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
                         "sample": f"{n} of {len(seqs_all)} sequences per step (append + fp64 attention)"},
        "e2e": {"value": round(gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------- ours
def run_ours(args):
    import torch

    rank, world, dist = dist_setup(args.gpus)
    dev = torch.device("cuda", torch.cuda.current_device())
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import paged_kv_cache_321_b200 as K
    from workloads import SPECS, make_workload

    spec = SPECS[args.workload]
    from paged_kv_cache_321_b200 import replicas

    wl = make_workload(spec, seed_offset=replicas.replica_seed_offset(spec.seed_offset, rank))
    sp = wl.spec
    stream = torch.cuda.current_stream()

    pool = K.Pool(sp.num_layers, sp.Hkv, sp.D, sp.bs, wl.max_seq_len, wl.num_blocks, sp.kv_dtype, device=dev)
    pool.k.copy_(torch.from_numpy(wl.pool_k.view(np.int16)))
    pool.v.copy_(torch.from_numpy(wl.pool_v.view(np.int16)))
    attn = K.attn_config(sp.Hq, sp.Hkv, sp.D, float(np.float32(sp.theta)), sp.eps, sp.rope_dim, sp.rope_style,
                         sp.window)
    rope = torch.empty(wl.max_seq_len * (sp.rope_dim or sp.D), dtype=torch.float32, device=dev)
    K.rope_table_fill(attn, wl.max_seq_len, rope)
    g = lambda a: None if a is None else torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    # the step's per-step inputs live in one device buffer (256-byte aligned
    # views), so the end-to-end leg below moves them with one host->device copy
    step_inputs = [np.ascontiguousarray(a) for a in (wl.q, wl.k, wl.v, wl.tok_req, wl.positions, wl.block_tables,
                                                      wl.ctx)]
    offs, nbytes = [], 0
    for a in step_inputs:
        offs.append(nbytes)
        nbytes += (a.nbytes + 255) // 256 * 256
    h_pack = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
    for a, o in zip(step_inputs, offs):
        h_pack[o:o + a.nbytes].copy_(torch.from_numpy(a.view(np.uint8).reshape(-1)))
    d_pack = h_pack.to(dev)
    views = [d_pack[o:o + a.nbytes].view(torch.from_numpy(a[:0]).dtype).view(a.shape)
             for a, o in zip(step_inputs, offs)]
    q, k, v, tok_req, positions, bt, ctx = views
    qn, kn = g(wl.q_norm_w), g(wl.k_norm_w)
    dseq, pseq = wl.decode_seqs, wl.prefill_seqs
    T = wl.T
    q_out = torch.empty((T, sp.Hq * sp.D), dtype=torch.float32, device=dev)
    kv_bytes = wl.kv_read_bytes()  # the decode sequences' K/V
    # decode inputs: the decode sequences' rows (views when they are all sequences)
    B = len(dseq)
    mx = int(wl.ctx[dseq].max(initial=0))
    def run_of(idx):
        """(start, stop) when idx is one run of consecutive integers, else None."""
        idx = np.asarray(idx, dtype=np.int64)
        if len(idx) and np.array_equal(idx, np.arange(idx[0], idx[0] + len(idx))):
            return int(idx[0]), int(idx[0]) + len(idx)
        return None

    def sel(t, idx):
        """Rows idx of t: a view when they are consecutive, else a gathered copy
        made once, outside the timed steps."""
        run = run_of(idx)
        if run is not None:
            return t[run[0]:run[1]]
        return t.index_select(0, torch.from_numpy(np.asarray(idx, dtype=np.int64)).to(dev)).contiguous()

    d_bt, d_ctx = sel(bt, dseq), sel(ctx, dseq)
    q3 = q_out.view(T, sp.Hq, sp.D)
    d_run = run_of(wl.cu_q[dseq])
    d_rows = torch.from_numpy(wl.cu_q[dseq].astype(np.int64)).to(dev)
    d_q = q3[d_run[0]:d_run[1]] if d_run else torch.empty((B, sp.Hq, sp.D), dtype=torch.float32, device=dev)
    out = torch.empty((B, sp.Hq, sp.D), dtype=torch.float32, device=dev)
    ws_n = K.decode_workspace_size(pool, attn, B, mx, args.split_tokens)
    ws = torch.zeros(ws_n // 4 + 64, dtype=torch.float32, device=dev)
    # prefill inputs: the chunk sequences' rows
    prefill_flops = 0
    if len(pseq):
        p_rows = np.concatenate([np.arange(wl.cu_q[r], wl.cu_q[r + 1]) for r in pseq]).astype(np.int64)
        p_rows_t = torch.from_numpy(p_rows).to(dev)
        p_run = run_of(p_rows)
        p_cu = np.zeros(len(pseq) + 1, dtype=np.int32)
        p_cu[1:] = np.cumsum(wl.q_lens[pseq])
        p_cu_t = torch.from_numpy(p_cu).to(dev)
        p_bt, p_ctx = sel(bt, pseq), sel(ctx, pseq)
        p_q = q3[p_run[0]:p_run[1]] if p_run else torch.empty((len(p_rows), sp.Hq, sp.D), dtype=torch.float32,
                                                               device=dev)
        p_out = torch.empty_like(p_q)
        p_maxq = int(wl.q_lens[pseq].max())
        seen = wl.positions[p_rows].astype(np.int64) + 1  # causal (query, key) pairs
        if sp.window > 0:
            seen = np.minimum(seen, sp.window)
        pairs = int(seen.sum())
        prefill_flops = pairs * sp.Hq * sp.D * 4  # QK^T and PV, 2 flops per multiply-add

    def append():
        K.kv_append(pool, sp.layer, attn, q, k, v, tok_req, positions, bt, q_out, qn, kn, rope, wl.max_seq_len,
                    stream=stream)

    def gather_q():
        # the workloads put each kind of sequence in one run, so the queries
        # are views of kv_append's output and nothing runs here; a layout
        # without runs would gather them with torch (not counted as ours)
        if B and not d_run:
            torch.index_select(q3, 0, d_rows, out=d_q)
        if prefill_flops and not p_run:
            torch.index_select(q3, 0, p_rows_t, out=p_q)

    def prefill():
        if prefill_flops:
            K.paged_prefill_attention(pool, sp.layer, attn, p_q, p_cu_t, p_ctx, p_bt, p_maxq, p_out, stream=stream)

    def decode():
        if B:
            K.paged_decode_attention(pool, sp.layer, attn, d_q, d_bt, d_ctx, mx, out, ws, args.split_tokens,
                                     stream=stream)

    def barrier():
        if dist is not None:
            dist.barrier()

    # ---- device-resident timing
    def step(i=None):
        append()
        gather_q()
        if prefill_flops:
            if i is not None:
                evp[i][0].record(stream)
            prefill()
            if i is not None:
                evp[i][1].record(stream)
        if i is not None:
            ev[i][0].record(stream)
        decode()
        if i is not None:
            ev[i][1].record(stream)

    for _ in range(max(args.warmup, 3)):
        step()
    pool.sync_status(stream)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    evp = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    clocks = ClockSampler(dev.index)
    clocks.start()
    # (1) K steps back to back, events only around the whole run: the kernels
    # of a step are launched with programmatic dependencies, and an event
    # recorded between two of them would stop the next one's launch from
    # overlapping the previous one, so per-kernel events stay out of this run
    barrier()
    torch.cuda.synchronize()
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for i in range(args.steps):
        step()
    t_end.record(stream)
    torch.cuda.synchronize()
    barrier()
    # (2) the same K steps with events around every decode and prefill launch:
    # the kernels' own durations for the roofline
    for i in range(args.steps):
        step(i)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    pool.sync_status(stream)
    step_ms = t_start.elapsed_time(t_end) / args.steps
    dec_ms = float(np.mean([a.elapsed_time(b) for a, b in ev]))
    pre_ms = float(np.mean([a.elapsed_time(b) for a, b in evp])) if prefill_flops else 0.0
    step_ms, dec_ms, pre_ms = replicas.max_over_ranks([step_ms, dec_ms, pre_ms], dist, dev)

    # ---- end to end through the C ABI with host buffers: H2D of the step's
    # inputs from pinned memory, the step, D2H of the attention output
    # (q, k, v, token -> sequence, positions, block tables and context lengths
    # in one pinned buffer, one copy; the decode output back)
    h_out = torch.empty(out.shape, dtype=torch.float32).pin_memory()
    h2d = sum(a.nbytes for a in step_inputs)
    d2h = h_out.numel() * h_out.element_size()
    e2e_steps = max(1, min(args.steps, 500))

    def e2e_step():
        d_pack.copy_(h_pack, non_blocking=True)
        step()
        h_out.copy_(out, non_blocking=True)

    for _ in range(3):
        e2e_step()
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    (e2e_ms,) = replicas.max_over_ranks([e2e_ms], dist, dev)
    pool.sync_status(stream)

    peak, peak_kind = measured_peaks()
    total_bytes = kv_bytes * world
    value = replicas.job_throughput(kv_bytes, world, step_ms * 1e-3) / 1e9
    achieved = kv_bytes / (dec_ms * 1e-3) / 1e9
    # where sequences share prefix blocks, HBM moves each physical slot once
    # (the repeats come from L2): the roofline uses those unique bytes
    kv_unique = wl.unique_kv_read_bytes() if sp.share_group else kv_bytes
    achieved_hbm = kv_unique / (dec_ms * 1e-3) / 1e9
    d_ctx_np = wl.ctx[dseq].astype(np.int64)
    moved = {"kv": kv_bytes, "kv_unique": kv_unique, "q": B * sp.Hq * sp.D * 4, "out": B * sp.Hq * sp.D * 4,
             "block_tables": int(((d_ctx_np + sp.bs - 1) // sp.bs).sum()) * 4, "ctx_lens": B * 4,
             "append_read": T * (sp.Hq + 2 * sp.Hkv) * sp.D * 4 + T * 8,
             "append_write": T * sp.Hq * sp.D * 4 + T * 2 * sp.Hkv * sp.D * 2}
    decode_launches = 2 if sp.Hq // sp.Hkv == 8 else 1  # groups of 8 add the merge grid
    traffic = ncu_traffic(args.workload)
    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(step_ms, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": sp.kv_dtype,
        "data": "synthetic",
        "config": {"workload": args.workload, "batch": B, "Hq": sp.Hq, "Hkv": sp.Hkv, "head_dim": sp.D,
                   "block_size": sp.bs, "kv_dtype": sp.kv_dtype, "ctx_range": [int(wl.ctx[dseq].min()) if B else 0, mx],
                   "kv_bytes_per_step": kv_bytes, "kv_unique_bytes_per_step": kv_unique,
                   "split_tokens": args.split_tokens or "auto",
                   "l2": f"inputs larger than L2 ({kv_bytes / 1e6:.0f} MB of K/V per step vs 126 MB L2)",
                   "parallelism": f"replicas x{world}"},
        "seq_steps_per_s": round(B * world / (step_ms * 1e-3), 1),
        "decode_attention_gbs": round(achieved * world, 2),
        "decode_attention_gbs_unique": round(achieved_hbm * world, 2),
        "pct_of_measured_hbm": round(100 * achieved_hbm / peak, 2),
        "pct_of_nominal_8tbs": round(100 * achieved_hbm / NOMINAL_HBM_GBS, 2),
        "moved_bytes_per_step": moved,
        "decode_us": round(dec_ms * 1e3, 2),
        "append_us_incl_gap": round((step_ms - dec_ms) * 1e3, 2),
        "roofline": {"bound": "hbm", "achieved": round(achieved_hbm, 2), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved_hbm / peak, 4), "traffic": traffic,
                     "peak_kind": peak_kind, "kernel": decode_kernel_name(sp)},
        "clocks": clk,
        "e2e": {"value": round(total_bytes / (e2e_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 5)},
        "gpu_launches": (1 + decode_launches + (1 if prefill_flops else 0)) * args.steps,  # append, decode, prefill
    }
    if prefill_flops:
        bf16_peak = measured_bf16_tflops()
        tf = prefill_flops / (pre_ms * 1e-3) / 1e12
        line["prefill"] = {"kernel": "kvp::pre::prefill_kernel", "us": round(pre_ms * 1e3, 2),
                           "flops_per_launch": prefill_flops, "tflops": round(tf, 2),
                           "roofline": {"bound": "tensor", "achieved": round(tf, 2), "peak": bf16_peak[0],
                                        "unit": "TFLOP/s", "frac": round(tf / bf16_peak[0], 4),
                                        "peak_kind": bf16_peak[1] + " bf16 (the fp16 dense rate is the same)"}}
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not prefill_flops:
        line["cpu_baseline"] = cpu_baseline(wl)
        line["cpu_baseline_single_thread"] = cpu_baseline(wl, budget_s=4.0, threads=1)
    if rank == 0:
        print(json.dumps(line), flush=True)
    pool.close()
    if dist is not None:
        dist.destroy_process_group()


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
