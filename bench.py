#!/usr/bin/env python
"""Benchmark of the KDA core on B200.

Workload (one step = one pass of the prefill hot path over one batch): B=1 sequence of
T=4096 tokens, H=32 heads, head_dim 128, 64-token chunks, BF16-exact inputs widened to
FP32, initial state N(0, 0.1): kda_gate (g_raw -> gate), kda_beta (b_logit -> beta) and
kda_chunk_prefill (q, k, v, gate, beta, state -> core, state). `--prefill-impl graw` runs
kda_beta + kda_chunk_prefill_graw instead (the gate formed inside the chunked kernels from
BF16 g_raw), `simt` the CUDA-core prefill.
Inputs are resident in HBM; L2 is flushed (a 512 MB write) before every timed step,
outside the timed events.
Multi-GPU: each rank runs its own independent sequence (weak scaling, no collective).

Also reported: the dominant kernel's roofline (CUDA events around each launch), a decode
leg (256 sequences x 1 token, kda_decode_fused, state GB/s), the same prefill in the
fused-input mode (kda_chunk_prefill_fused on BF16 rows), an end-to-end leg through
kda_chunk_prefill_host from pinned host buffers (copies inside the timed region), the block
(prefill with a per-stage split, its GEMM, block decode), 4 streams x 65500 tokens of prefill
(inputs larger than L2), and the
FP64 oracle timed on the host cores (`cpu_baseline`). `--impl reference` times the oracle
alone (it is this project's reference implementation) and prints its own line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "KDA prefill tokens/s (% tensor-core roofline); decode state GB/s (% of HBM peak)"
B, T, H, D = 1, 4096, 32, 128
CONFIG = {"workload": "kda_chunk_prefill B1 T4096 H32 D128 chunk64 (gate+beta+chunked core), FP32 I/O",
          "global_batch": B, "seq_len": T, "heads": H, "head_dim": D, "chunk": 64,
          "l2": "flushed before every timed step (512 MB write)"}
# Algorithmic bytes per token-head of the timed chunked call: q, k, v, core at D FP32 values
# each + beta, and the gate input: D BF16 g_raw values (graw) or D FP32 gate values (tc, simt).
BYTES_PER_TOKEN_HEAD = {"graw": 4 * D * 4 + D * 2 + 4, "tc": 5 * D * 4 + 4, "simt": 5 * D * 4 + 4}
# kernels one step launches: beta + intra, fix-up, state (graw); + gate (tc); gate, beta, one (simt)
LAUNCHES_PER_STEP = {"graw": 4, "tc": 5, "simt": 3}
FLOPS_PER_TOKEN_HEAD = 139_000  # L, M, WY/UT solve, W.S, Q.S, M.U, K^T.U at C=64, D=128 (triangles as half)


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), float(j["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, "fallback"


def _src_sha(rel):
    with open(os.path.join(ROOT, rel), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def _traffic(kernel_key):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on this source."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        j = json.load(f).get(kernel_key)
    if not j or j.get("src_sha") != _src_sha(j["src"]):
        return None
    return j.get("dram_bytes_per_launch")


class Clocks:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            time.sleep(1.0)  # nvidia-smi start-up; the first sample lands before the warm-up
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.out = ""
        if self.proc:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = [r.split(",") for r in (getattr(self, "out", "") or "").strip().splitlines() if r.strip()]
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
                for n, v in zip(names, r[5:9]):
                    if v.strip().lower() == "active":
                        reasons.add(n)
            except (ValueError, IndexError):
                pass
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def _cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def _oracle_baseline(T_sample):
    """The FP64 oracle (as it stands) on the first T_sample tokens of the workload: gate,
    sigmoid and the token recurrence for all 32 heads, on all host cores."""
    import oracle
    from synth import core_inputs
    ci = core_inputs(1, T_sample, H, D, seed=1, bf16_inputs=True, s0_std=0.1)
    cores = oracle.default_threads()
    oracle.build()
    t0 = time.perf_counter()
    g = oracle.gate(ci.g_raw.float(), ci.dt_bias, ci.a_log, H, D)
    beta = oracle.sigmoid(ci.b_logit)
    oracle.recurrence(ci.q, ci.k, ci.v, g, beta, ci.s0, 1.0, cores)
    dt = time.perf_counter() - t0
    return T_sample / dt, dt, cores


def run_reference(args, rank, world):
    if rank != 0:
        return 0
    T_sample = 512
    times = []
    for i in range(args.warmup + args.steps):
        tps, dt, cores = _oracle_baseline(T_sample)
        if i >= args.warmup:
            times.append(dt)
    ms = 1000.0 * sum(times) / len(times)
    value = T_sample / (ms / 1000.0)
    sample = f"oracle on the first {T_sample} tokens of the T=4096 sequence, all 32 heads, per step"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": dict(CONFIG, parallelism=f"dp{world}", prefill_impl=args.prefill_impl),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--prefill-impl", default="tc", choices=["tc", "graw", "simt"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-block", action="store_true", help="skip the block-prefill leg")
    ap.add_argument("--no-long", action="store_true", help="skip the 4 x 65500-token prefill leg")
    args = ap.parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)
    assert args.warmup >= 3, "at least 3 warm-up steps"

    import torch
    import torch.distributed as dist
    import kda_gated_delta_gate_b200 as kda
    from synth import core_inputs, pad_rows, t_pad

    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", init_method="env://", timeout=__import__("datetime").timedelta(seconds=120))
    dev = torch.device("cuda", local)
    kda.lib()
    stream = torch.cuda.current_stream(dev)
    s = stream.cuda_stream
    d = kda.dims(H, D)
    Tp = t_pad(T)

    # ---- inputs resident in HBM (each rank its own sequence: seed differs by rank)
    ci = core_inputs(B, T, H, D, seed=1 + 1000 * rank, bf16_inputs=True, s0_std=0.1)
    q = pad_rows(ci.q, Tp, 0.0).to(dev)
    k = pad_rows(ci.k, Tp, 0.0).to(dev)
    v = pad_rows(ci.v, Tp, 0.0).to(dev)
    g_raw = pad_rows(ci.g_raw, Tp, 0.0).to(dev)
    b_logit = pad_rows(ci.b_logit, Tp, 0.0).to(dev)
    dt_bias, a_log = ci.dt_bias.to(dev), ci.a_log.to(dev)
    gate = torch.empty((B * Tp, H, D), device=dev)
    beta = torch.empty((B * Tp, H), device=dev)
    core = torch.empty((B * Tp, H, D), device=dev)
    s0_dev = ci.s0[0].to(dev)
    state = s0_dev.clone()
    ptrs = kda.ptr_array([state], device=dev)
    scratch = torch.empty(max(16, kda.kda_chunk_prefill_scratch_bytes(B, T, d)), dtype=torch.uint8, device=dev)
    flush = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    ev_k = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    ev_s = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]

    graw = args.prefill_impl == "graw"

    def step(kev=None):
        if not graw:
            kda.kda_gate(g_raw, dt_bias, a_log, gate, B * T, d, s)
        kda.kda_beta(b_logit, beta, B * T * H, s)
        if kev:
            kev[0].record(stream)
        if graw:
            kda.kda_chunk_prefill_graw(q, k, v, g_raw, dt_bias, a_log, beta, ptrs, core, B, T, d, s, scratch=scratch)
        else:
            kda.kda_chunk_prefill(q, k, v, gate, beta, ptrs, core, B, T, d, s, impl=args.prefill_impl,
                                  scratch=scratch)
        if kev:
            kev[1].record(stream)
        return LAUNCHES_PER_STEP[args.prefill_impl]

    launches = 0
    with Clocks(local) as clk:
        for _ in range(args.warmup):
            state.copy_(s0_dev)
            flush.zero_()
            step()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        for i in range(args.steps):
            state.copy_(s0_dev)  # every timed step starts from the workload's initial state
            flush.zero_()
            ev_s[i][0].record(stream)
            launches += step(ev_k[i])
            ev_s[i][1].record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    step_ms = sum(a.elapsed_time(b) for a, b in ev_s) / args.steps
    kern_all = [a.elapsed_time(b) for a, b in ev_k]
    kern_ms = sum(kern_all) / args.steps
    kern_med, kern_min = statistics.median(kern_all), min(kern_all)
    if world > 1:
        t = torch.tensor([step_ms, kern_ms], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        step_ms, kern_ms = t.tolist()

    hbm, tc_peak, peak_kind = _peaks()
    alg_bytes = B * T * H * BYTES_PER_TOKEN_HEAD[args.prefill_impl] + 2 * B * H * D * D * 4
    alg_flops = B * T * H * FLOPS_PER_TOKEN_HEAD
    achieved_gbs = alg_bytes / (kern_ms * 1e-3) / 1e9
    achieved_tf = alg_flops / (kern_ms * 1e-3) / 1e12

    # ---- decode leg: 256 sequences x 1 token, fused stateful row (state GB/s)
    dec = _decode_leg(kda, torch, dev, s, stream, flush, hbm)

    # ---- the same workload in the fused-input mode (BF16 q|k|v rows + g_raw, gate in-kernel)
    fused = _fused_leg(kda, torch, dev, s, stream, flush, d, ci, Tp, hbm, tc_peak, scratch)

    # ---- end-to-end legs from pinned host buffers, copies timed: the headline call (FP32 I/O)
    # and the serving layout (BF16 q|k|v rows)
    e2e = _e2e_leg(kda, torch, dev, s, stream, d, args, ci, Tp, world, scratch, "f32")
    e2e_bf16 = _e2e_leg(kda, torch, dev, s, stream, d, args, ci, Tp, world, scratch, "bf16", seg=512)

    # ---- the full block (projections + front end + core + back end) and its dominant GEMM
    blk = None if args.no_block else _block_leg(kda, torch, dev, s, stream, flush, tc_peak, hbm)

    # ---- long multi-stream prefill: 4 streams x 65500 tokens (T_pad 65536)
    del q, k, v, g_raw, b_logit, gate, beta, core, scratch
    torch.cuda.empty_cache()
    long_leg = None if args.no_long else _long_leg(kda, torch, dev, s, stream, hbm, tc_peak, rank)

    result = None
    if rank == 0:
        tokens_per_s = world * B * T / (step_ms * 1e-3)
        cpu = None
        if not args.no_cpu_baseline:
            tps, dt, cores = _oracle_baseline(T)
            cpu = {"value": tps, "unit": "tokens/s", "cores": cores, "kind": "oracle", "cpu_model": _cpu_model(),
                   "sample": f"FP64 oracle (gate, sigmoid, token recurrence, 32 heads) over the whole {T}-token "
                             f"workload once; {dt:.2f} s wall on {cores} threads"}
        result = {
            "metric": METRIC, "value": tokens_per_s, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic", "config": dict(CONFIG, parallelism=f"dp{world}",
                                                                                     prefill_impl=args.prefill_impl),
            "roofline": {"kernel": "kda_chunk_prefill_graw" if graw else "kda_chunk_prefill", "bound": "hbm", "achieved": achieved_gbs, "peak": hbm,
                         "unit": "GB/s", "frac": achieved_gbs / hbm, "peak_kind": peak_kind,
                         "traffic": _traffic("chunk_prefill_" + args.prefill_impl),
                         "kernel_ms": kern_ms, "kernel_ms_median": kern_med, "kernel_ms_min": kern_min,
                         "alg_bytes_per_launch": alg_bytes,
                         "tensor": {"achieved": achieved_tf, "peak": tc_peak, "unit": "TFLOP/s",
                                    "frac": achieved_tf / tc_peak, "alg_flops_per_launch": alg_flops}},
            "decode": dec,
            "fused_input": fused,
            "block_prefill": blk,
            "long_prefill": long_leg,
            "e2e": e2e,
            "e2e_bf16_host": e2e_bf16,
            "cpu_baseline": cpu,
            "gpu_launches": launches,
            "clocks": clk.summary(),
        }
        print(json.dumps(result), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def _decode_leg(kda, torch, dev, s, stream, flush, hbm):
    from synth import decode_inputs
    N = 256
    di = decode_inputs(N, H, D, seed=3, device="cpu")
    dd = kda.dims(H, D)
    x, cw, gr = di.x.to(dev), di.conv_w.to(dev), di.g_raw.to(dev)
    dtb, al, bl, og, ow = di.dt_bias.to(dev), di.a_log.to(dev), di.b_logit.to(dev), di.out_gate.to(dev), di.o_norm.to(dev)
    cs = [di.conv_state[n].to(dev).clone() for n in range(N)]
    hs = [di.s0[n].to(dev).clone() for n in range(N)]
    cp, hp = kda.ptr_array(cs, device=dev), kda.ptr_array(hs, device=dev)
    out = torch.empty((N, H * D), dtype=torch.bfloat16, device=dev)
    times = []
    for i in range(25):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        kda.kda_decode_fused(x, cp, cw, gr, dtb, al, bl, hp, og, ow, out, None, None, N, dd, s)
        b.record(stream)
        torch.cuda.synchronize()
        if i >= 5:
            times.append(a.elapsed_time(b))
    ms = statistics.median(times)
    state_bytes = N * H * D * D * 4 * 2
    all_bytes = state_bytes + N * (3 * H * D * 2 + 3 * H * D * 3 * 2 * 2 + H * D * 2 * 3 + H * 4)
    return {"workload": "kda_decode_fused 256 seqs x 1 token, H32 D128 (conv+gate+beta+recurrence+o_norm)",
            "ms": ms, "tokens_per_s": N / (ms * 1e-3), "state_gbs": state_bytes / (ms * 1e-3) / 1e9,
            "all_gbs": all_bytes / (ms * 1e-3) / 1e9, "hbm_peak_gbs": hbm,
            "frac_hbm": all_bytes / (ms * 1e-3) / 1e9 / hbm}


def _block_leg(kda, torch, dev, s, stream, flush, tc_peak, hbm):
    """KDA block prefill, hidden 4096, H 32, D 128, rank 128, T 8192 (BF16 weights N(0, 0.02)),
    the q_proj-sized GEMM (8192 x 4096 x 4096) alone, and the block decode on the same
    weights: one token of one sequence, K = 4 rows of one sequence (decode_k), and 256
    sequences x 1 token."""
    import types
    from synth import block_hidden, block_weights
    hidden, Hh, Dd, rank, Tb = 4096, 32, 128, 128, 8192
    Wt = block_weights(hidden, Hh, Dd, rank, seed=2, device=dev)
    hid = block_hidden(Tb, hidden, seed=2, device=dev)
    dw = types.SimpleNamespace(q_proj=Wt.w_q, k_proj=Wt.w_k, v_proj=Wt.w_v, conv=Wt.conv_w, f_a=Wt.f_a, f_b=Wt.f_b,
                               dt_bias=Wt.dt_bias, a_log=Wt.a_log, b_proj=Wt.b_proj, g_a=Wt.g_a, g_b=Wt.g_b,
                               o_norm=Wt.o_norm, o_proj=Wt.o_proj, hidden=hidden, rank=rank)
    st = kda.block_weights_struct(dw)
    ws = kda.Workspace(kda.dims(Hh, Dd), hidden, rank, max_tokens=Tb)
    hs = torch.zeros((Hh, Dd, Dd), device=dev)
    cs = torch.zeros((3 * Hh * Dd, 3), dtype=torch.bfloat16, device=dev)

    def timed(fn, reps=6, warm=3):
        ts = []
        for i in range(warm + reps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            torch.cuda.synchronize()
            if i >= warm:
                ts.append(a.elapsed_time(b))
        return statistics.median(ts)

    ms = timed(lambda: kda.kda_block_prefill(st, hid, Tb, hs, cs, 0.0, ws, s))
    qkv, cd = Hh * Dd, 3 * Hh * Dd
    stages = _block_stages(kda, torch, dev, s, stream, flush, Wt, hid, ws, Tb, hidden, Hh, Dd, rank)
    flops = 2.0 * Tb * hidden * (3 * qkv + 2 * rank + Hh) + 2.0 * Tb * rank * 2 * qkv + 2.0 * Tb * qkv * hidden
    C = torch.empty((Tb, hidden), dtype=torch.bfloat16, device=dev)
    gms = timed(lambda: kda.kda_gemm_bf16(hid, Wt.w_q, C, Tb, hidden, hidden, stream=s))
    gflop = 2.0 * Tb * hidden * hidden
    # block decode (L2 flushed before every call, so the weights stream from HBM)
    wbytes = 2.0 * (3 * qkv * hidden + 2 * rank * hidden + 2 * qkv * rank + Hh * hidden + qkv * hidden)
    sbytes = 2.0 * Hh * Dd * Dd * 4 + 2.0 * cd * 3 * 2  # one sequence's state + conv state, read + write
    g = torch.Generator(device=dev).manual_seed(3)
    n_b = 256
    hs_b = torch.randn((n_b, Hh, Dd, Dd), generator=g, device=dev) * 0.1
    cs_b = torch.randn((n_b, cd, 3), generator=g, device=dev).to(torch.bfloat16)
    ph1, pc1 = kda.ptr_array([hs_b[0]], device=dev), kda.ptr_array([cs_b[0]], device=dev)
    phn, pcn = kda.ptr_array(list(hs_b), device=dev), kda.ptr_array(list(cs_b), device=dev)
    ms1 = timed(lambda: kda.kda_block_decode(st, hid[:1], 1, ph1, pc1, ws, s))
    graph = kda.kda_block_decode_graph(st, hid[:1], 1, ph1, pc1, ws)  # the same call, replayed
    ms1g = timed(lambda: graph.launch(s))
    graph.close()
    msk = timed(lambda: kda.kda_block_decode_k(st, hid[:4], 4, hs_b[1], cs_b[1], [], [], ws, s))
    msn = timed(lambda: kda.kda_block_decode(st, hid[:n_b], n_b, phn, pcn, ws, s))
    dec = {"one_token": {"ms": ms1, "tokens_per_s": 1 / (ms1 * 1e-3),
                         "gbs": (wbytes + sbytes) / (ms1 * 1e-3) / 1e9,
                         "frac_hbm": (wbytes + sbytes) / (ms1 * 1e-3) / 1e9 / hbm},
           "one_token_graph": {"ms": ms1g, "tokens_per_s": 1 / (ms1g * 1e-3),
                               "frac_hbm": (wbytes + sbytes) / (ms1g * 1e-3) / 1e9 / hbm,
                               "call": "kda_block_decode_graph once, kda_graph_launch per step"},
           "decode_k4": {"ms": msk, "tokens_per_s": 4 / (msk * 1e-3),
                         "gbs": (wbytes + sbytes) / (msk * 1e-3) / 1e9},
           "batch256": {"ms": msn, "tokens_per_s": n_b / (msn * 1e-3),
                        "gbs": (wbytes + n_b * sbytes) / (msn * 1e-3) / 1e9,
                        "frac_hbm": (wbytes + n_b * sbytes) / (msn * 1e-3) / 1e9 / hbm},
           "weights_bytes": wbytes, "state_bytes_per_seq": sbytes}
    # packed sequences through one block call, the same 8192 rows: 8 x 1024 (batched) and a ragged mix (varlen)
    ws2 = kda.Workspace(kda.dims(Hh, Dd), hidden, rank, max_tokens=Tb, max_seqs=64)
    lens = [3000, 2000, 1500, 1000, 500, 192]
    cu = torch.tensor([0] + [sum(lens[:i + 1]) for i in range(len(lens))], dtype=torch.int32, device=dev)
    p8h, p8c = kda.ptr_array(list(hs_b[:8]), device=dev), kda.ptr_array(list(cs_b[:8]), device=dev)
    msb = timed(lambda: kda.kda_block_prefill_batched(st, hid, 8, Tb // 8, p8h, p8c, ws2, s))
    msv = timed(lambda: kda.kda_block_prefill_varlen(st, hid, cu, len(lens), (max(lens) + 63) // 64, Tb, p8h, p8c,
                                                     ws2, s))
    # batched speculative verify + accepted-row fold: N sequences x 4 draft rows, states left in place by the
    # verify (the fold then advances them)
    ver = {}
    for n_v in (8, 64):
        rows = 4 * n_v
        cu_v = torch.arange(0, rows + 1, 4, dtype=torch.int32, device=dev)
        acc_v = torch.full((n_v,), 2, dtype=torch.int32, device=dev)
        tabs = torch.empty(kda.kda_chunk_verify_tables_bytes(n_v, kda.dims(Hh, Dd)) // 4, device=dev)
        pvh, pvc = kda.ptr_array(list(hs_b[:n_v]), device=dev), kda.ptr_array(list(cs_b[:n_v]), device=dev)
        msv1 = timed(lambda: kda.kda_block_verify(st, hid[:rows], cu_v, n_v, rows, pvh, pvc, tabs, ws2, s))
        msf = timed(lambda: (kda.kda_block_verify(st, hid[:rows], cu_v, n_v, rows, pvh, pvc, tabs, ws2, s),
                             kda.kda_block_verify_fold(cu_v, acc_v, n_v, rows, tabs, pvh, pvc, ws2, s)))
        ver[f"n{n_v}_k4"] = {"verify_ms": msv1, "verify_and_fold_ms": msf, "draft_rows_per_s": rows / (msv1 * 1e-3),
                             "call": "kda_block_verify (+ kda_block_verify_fold, 2 rows accepted per sequence)"}
        del tabs
    ws2.close()
    packed = {"batched_8x1024": {"ms": msb, "tokens_per_s": Tb / (msb * 1e-3), "call": "kda_block_prefill_batched"},
              "varlen_ragged": {"ms": msv, "tokens_per_s": Tb / (msv * 1e-3), "lens": lens,
                                "call": "kda_block_prefill_varlen"}}
    del hs_b, cs_b
    ws.close()
    return {"workload": "kda_block_prefill hidden 4096 H32 D128 rank 128 T8192 (9 GEMMs + conv + gate + core + o_norm)",
            "ms": ms, "tokens_per_s": Tb / (ms * 1e-3), "proj_flops": flops,
            "tflops_all": flops / (ms * 1e-3) / 1e12,
            "stages_ms": stages,
            "gemm": {"shape": "8192x4096x4096 bf16->bf16", "ms": gms, "tflops": gflop / (gms * 1e-3) / 1e12,
                     "peak": tc_peak, "frac": gflop / (gms * 1e-3) / 1e12 / tc_peak},
            "block_decode": dec, "packed_prefill": packed, "verify": ver}


def _fused_leg(kda, torch, dev, s, stream, flush, d, ci, Tp, hbm, tc_peak, scratch):
    """The headline workload through kda_chunk_prefill_fused: BF16 q|k|v rows (the front end's
    conv_out layout) and BF16 g_raw in, the gate formed in the kernel, FP32 beta (kda_beta's
    output), FP32 core and state out; L2 flushed before every call. Algorithmic bytes per
    token-head: q, k, v and g_raw at D BF16 values each, beta 4 B, core D FP32 values."""
    from synth import pad_rows
    qkv = torch.cat([ci.q.reshape(B, T, H * D), ci.k.reshape(B, T, H * D), ci.v.reshape(B, T, H * D)], dim=-1)
    qkv = pad_rows(qkv.to(torch.bfloat16), Tp, 0.0).to(dev)
    g_raw = pad_rows(ci.g_raw, Tp, 0.0).to(dev)
    beta = pad_rows(ci.b_logit, Tp, 0.0).to(dev)
    kda.kda_beta(beta, beta, beta.numel(), s)
    dt_bias, a_log = ci.dt_bias.to(dev), ci.a_log.to(dev)
    s0_dev = ci.s0[0].to(dev)
    state = s0_dev.clone()
    ptrs = kda.ptr_array([state], device=dev)
    core = torch.empty((B * Tp, H, D), device=dev)
    ts = []
    for i in range(3 + 20):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        kda.kda_chunk_prefill_fused(qkv, g_raw, dt_bias, a_log, beta, ptrs, core, B, T, d, s, scratch=scratch)
        b.record(stream)
        torch.cuda.synchronize()
        if i >= 3:
            ts.append(a.elapsed_time(b))
    ms = statistics.median(ts)
    alg = B * T * H * (3 * D * 2 + D * 2 + 4 + D * 4) + 2 * B * H * D * D * 4
    flops = B * T * H * FLOPS_PER_TOKEN_HEAD
    return {"workload": "kda_chunk_prefill_fused B1 T4096 H32 D128 (BF16 q|k|v rows and g_raw in, FP32 core out)",
            "kernel_ms": ms, "tokens_per_s": B * T / (ms * 1e-3), "alg_bytes_per_launch": alg,
            "hbm_frac": alg / (ms * 1e-3) / 1e9 / hbm, "tensor_frac": flops / (ms * 1e-3) / 1e12 / tc_peak}


def _long_leg(kda, torch, dev, s, stream, hbm, tc_peak, rank):
    """kda_gate + kda_beta + kda_chunk_prefill on 4 equal-length streams of 65500 tokens (T_pad
    65536), H 32, D 128, FP32 I/O; the inputs (about 21 GB) are far larger than L2, so no flush."""
    from synth import core_inputs, pad_rows, t_pad
    Bl, Tl = 4, 65500
    d = kda.dims(H, D)
    Tp = t_pad(Tl)
    ci = core_inputs(Bl, Tl, H, D, seed=4 + 1000 * rank, bf16_inputs=True, s0_std=0.1, device=dev)
    q, k, v = (pad_rows(x, Tp, 0.0) for x in (ci.q, ci.k, ci.v))
    g_raw = pad_rows(ci.g_raw, Tp, 0.0)
    b_logit = pad_rows(ci.b_logit, Tp, 0.0)
    dt_bias, a_log = ci.dt_bias, ci.a_log
    states = [ci.s0[b].clone() for b in range(Bl)]
    del ci
    ptrs = kda.ptr_array(states, device=dev)
    gate = torch.empty((Bl * Tp, H, D), device=dev)
    beta = torch.empty((Bl * Tp, H), device=dev)
    core = torch.empty((Bl * Tp, H, D), device=dev)
    scratch = torch.empty(kda.kda_chunk_prefill_scratch_bytes(Bl, Tl, d), dtype=torch.uint8, device=dev)
    steps, kms = [], []
    for i in range(3 + 5):
        e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        e[0].record(stream)
        kda.kda_gate(g_raw, dt_bias, a_log, gate, Bl * Tp, d, s)
        kda.kda_beta(b_logit, beta, Bl * Tp * H, s)
        e[1].record(stream)
        kda.kda_chunk_prefill(q, k, v, gate, beta, ptrs, core, Bl, Tl, d, s, scratch=scratch)
        e[2].record(stream)
        torch.cuda.synchronize()
        if i >= 3:
            steps.append(e[0].elapsed_time(e[2]))
            kms.append(e[1].elapsed_time(e[2]))
    ms, kern = statistics.median(steps), statistics.median(kms)
    alg = Bl * Tl * H * BYTES_PER_TOKEN_HEAD["tc"] + 2 * Bl * H * D * D * 4
    flops = Bl * Tl * H * FLOPS_PER_TOKEN_HEAD
    del q, k, v, g_raw, b_logit, gate, beta, core, scratch, states
    torch.cuda.empty_cache()
    return {"workload": "kda_gate + kda_beta + kda_chunk_prefill, 4 streams x 65500 tokens (T_pad 65536), H32 D128, "
                        "FP32 I/O; inputs larger than L2",
            "ms_per_step": ms, "tokens_per_s": Bl * Tl / (ms * 1e-3), "kernel_ms": kern,
            "hbm_frac": alg / (kern * 1e-3) / 1e9 / hbm, "tensor_frac": flops / (kern * 1e-3) / 1e12 / tc_peak,
            "alg_bytes": alg}


def _block_stages(kda, torch, dev, s, stream, flush, Wt, hid, ws, Tb, hidden, Hh, Dd, rank, reps=6):
    """The block prefill's stages, run one after another through their own C-ABI calls on the
    block's workspace (the order and arguments kda_block_prefill uses), with CUDA events between
    them: median ms per stage over `reps` runs, L2 flushed before each run."""
    bf = torch.bfloat16
    qkv, cd = Hh * Dd, 3 * Hh * Dd
    d = kda.dims(Hh, Dd)
    qp = ws.view("qkv_proj", (Tb, cd), bf)
    co = ws.view("conv_out", (Tb, cd), bf)
    fa = ws.view("f_a_out", (Tb, rank), bf)
    gr = ws.view("g_raw", (Tb, qkv), bf)
    be = ws.view("beta", (Tb, Hh), torch.float32)
    core = ws.view("core", (Tb, Hh, Dd), torch.float32)
    ga = ws.view("g_a_out", (Tb, rank), bf)
    og = ws.view("out_gate", (Tb, qkv), bf)
    on = ws.view("o_norm_out", (Tb, qkv), bf)
    fo = ws.view("final_out", (Tb, hidden), bf)
    sc_ptr, sc_bytes = ws.buffer("prefill_scratch")
    scratch = kda._device_view(sc_ptr, (sc_bytes,), torch.uint8)
    hs = torch.zeros((Hh, Dd, Dd), device=dev)
    cs = torch.zeros((cd, 3), dtype=bf, device=dev)
    hp = kda.ptr_array([hs], device=dev)
    gemm = lambda A, W, C, N, K: kda.kda_gemm_bf16(A, W, C, Tb, N, K, stream=s)
    stages = (
        ("proj_qkv", lambda: [gemm(hid, w, qp[:, i * qkv:(i + 1) * qkv], qkv, hidden)
                              for i, w in enumerate((Wt.w_q, Wt.w_k, Wt.w_v))]),
        ("front_conv_silu_l2", lambda: kda.kda_front_conv_silu_l2(qp, cs, Wt.conv_w, co, None, None, None, 0.0, Tb,
                                                                   d, s)),
        ("gate_beta_inputs", lambda: (gemm(hid, Wt.f_a, fa, rank, hidden), gemm(fa, Wt.f_b, gr, qkv, rank),
                                      gemm(hid, Wt.b_proj, be, Hh, hidden), kda.kda_beta(be, be, Tb * Hh, s))),
        ("core_prefill_fused", lambda: kda.kda_chunk_prefill_fused(co, gr, Wt.dt_bias, Wt.a_log, be, hp, core, 1, Tb,
                                                                   d, s, scratch=scratch)),
        ("out_gate_norm_oproj", lambda: (gemm(hid, Wt.g_a, ga, rank, hidden), gemm(ga, Wt.g_b, og, qkv, rank),
                                         kda.kda_back_gated_rmsnorm(core, og, Wt.o_norm, on, Tb, d, s),
                                         gemm(on, Wt.o_proj, fo, hidden, qkv))),
    )
    times = {name: [] for name, _ in stages}
    for i in range(3 + reps):
        flush.zero_()
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(len(stages) + 1)]
        evs[0].record(stream)
        for j, (_, fn) in enumerate(stages):
            fn()
            evs[j + 1].record(stream)
        torch.cuda.synchronize()
        if i >= 3:
            for j, (name, _) in enumerate(stages):
                times[name].append(evs[j].elapsed_time(evs[j + 1]))
    return {name: statistics.median(t) for name, t in times.items()}


def _pcie(torch, dev, stream, nbytes=256 << 20):
    """Measured pinned-host <-> device copy bandwidth (GB/s), each direction alone: the floor
    of an end-to-end call is its larger direction's bytes over these."""
    h = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
    g = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    out = {}
    for name, fn in (("h2d_gbs", lambda: g.copy_(h, non_blocking=True)),
                     ("d2h_gbs", lambda: h.copy_(g, non_blocking=True))):
        fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(3):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        out[name] = 3 * nbytes / (a.elapsed_time(b) * 1e-3) / 1e9
    return out


def _e2e_leg(kda, torch, dev, s, stream, d, args, ci, Tp, world, scratch, mode="f32", seg=1024):
    """The headline prefill through the public C ABI from pinned host buffers, the copies inside
    the timed region, segment by segment with the copies of one segment overlapping the kernels
    of the next.
    mode "f32": kda_chunk_prefill_host_f32, the same kernels and inputs as the timed step (FP32
    q, k, v; BF16 g_raw; FP32 beta logits; kda_gate + kda_beta + kda_chunk_prefill).
    mode "bf16": kda_chunk_prefill_host, the serving layout (BF16 q|k|v rows as the front end
    writes them, the gate formed in the core). Both return the FP32 core rows and final state."""
    pcie = _pcie(torch, dev, stream)
    qf, kf, vf = (x[0].reshape(T, H * D).contiguous() for x in (ci.q, ci.k, ci.v))
    if mode == "f32":
        host = {"q": qf.pin_memory(), "k": kf.pin_memory(), "v": vf.pin_memory()}
        nbytes = kda.kda_chunk_prefill_host_f32_bytes(T, seg, d)
    else:
        host = {"qkv": torch.cat([qf, kf, vf], dim=-1).to(torch.bfloat16).contiguous().pin_memory()}
        nbytes = kda.kda_chunk_prefill_host_bytes(T, seg, d)
    host["g_raw"] = ci.g_raw[0].contiguous().pin_memory()
    host["b_logit"] = ci.b_logit[0].contiguous().pin_memory()
    state_h = ci.s0[0].clone().pin_memory()
    core_h = torch.empty((T, H, D)).pin_memory()
    dt_bias, a_log = ci.dt_bias.to(dev), ci.a_log.to(dev)
    buf = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    h2d = sum(t.numel() * t.element_size() for t in host.values()) + state_h.numel() * 4
    d2h = core_h.numel() * 4 + state_h.numel() * 4

    def one():
        if mode == "f32":
            kda.kda_chunk_prefill_host_f32(host["q"], host["k"], host["v"], host["g_raw"], host["b_logit"], dt_bias,
                                           a_log, state_h, core_h, T, seg, buf, d, s)
        else:
            kda.kda_chunk_prefill_host(host["qkv"], host["g_raw"], host["b_logit"], dt_bias, a_log, state_h, core_h,
                                       T, seg, buf, d, s)

    for _ in range(3):
        one()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n = max(3, args.steps // 2)
    a.record(stream)
    for _ in range(n):
        one()
    b.record(stream)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / n
    if world > 1:
        import torch.distributed as dist
        t = torch.tensor([ms], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = t.item()
    ins = ("FP32 q, k, v, BF16 g_raw, FP32 beta logits and state in" if mode == "f32" else
           "BF16 q|k|v rows, BF16 g_raw, FP32 beta logits and state in")
    call = "kda_chunk_prefill_host_f32" if mode == "f32" else "kda_chunk_prefill_host"
    return {"value": world * B * T / (ms * 1e-3), "unit": "tokens/s", "ms_per_step": ms,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "pcie_floor_ms": max(h2d / pcie["h2d_gbs"], d2h / pcie["d2h_gbs"]) / 1e6,
            "pcie": pcie,
            "call": f"{call}, {seg}-token segments ({ins}; FP32 core and state out; copies and kernels of "
                    "consecutive segments overlapped)"}


if __name__ == "__main__":
    sys.exit(main())
