"""Benchmark of the TurboQuant KV-cache hot path on B200 (one JSON line on stdout).

One step = one pass of the whole path over one batch of synthetic input:
  1. encode a Llama-8B-shaped KV block: K, V bf16 [8 heads x 32768 tokens x d=128] (2% outlier
     channels x20, log-normal token norms); keys Algorithm 1 at 3 bits, values Algorithm 2 at 3 bits;
  2. decode that block back to fp32 (the round trip);
  3. one decode-attention step over the resident packed cache of the decode-attention workload:
     batch 16, 32 query / 8 KV heads, d=128, 131072 cached tokens (keys Algorithm 1 at 3 bits,
     values Algorithm 2 at 2 bits), bf16 queries.
Throughput unit: KV vectors per second through the path (encoded + decoded + attended key/value
vectors; an attended token-head counts its key and its value). Inputs are larger than L2.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU (torchrun, one process per GPU): every rank runs the same step on its own data (weak
scaling, no collective on the data path); the step time is the max over ranks.
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

METRIC = "encode vectors/s + packed-KV decode-attention tokens/s, as % of B200 HBM roofline"
UNIT = "vectors/s"

# workload sizes
D = 128
BLK_HEADS, BLK_TOKENS = 8, 32768                 # Llama-8B-shaped block
ATT_B, ATT_HQ, ATT_HKV, ATT_T = 16, 32, 8, 131072  # decode-attention cache
K_BITS, V_BITS_BLOCK, V_BITS_CACHE = 3, 3, 2

# algorithmic HBM bytes per unit (read + write of the data the kernel must touch)
G = D // 32
B_ENC_K = 2 * D + K_BITS * D // 8 + 2                        # bf16 in, codes + fp16 norm out
B_ENC_V = 2 * D + (V_BITS_BLOCK - 1) * D // 8 + D // 8 + 4   # bf16 in, codes + signs + norm + gamma
B_DEC_K = K_BITS * D // 8 + 2 + 4 * D                        # packed in, fp32 out
B_DEC_V = (V_BITS_BLOCK - 1) * D // 8 + D // 8 + 4 + 4 * D
B_ATT_TOKEN_HEAD = (K_BITS * D // 8 + 2) + ((V_BITS_CACHE - 1) * D // 8 + D // 8 + 4)   # 86 bytes


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "20"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 6:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[2:6]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------------------------------------
# reference arm: the oracle on the host cores, a bounded sample of the same workload
# ------------------------------------------------------------------------------------------------

def oracle_step(sample):
    """One bounded oracle step: encode + decode `n` block vectors of K and V, attention of one
    (batch, KV head) slice of `t` cached tokens for its 4 query heads. Returns vectors processed."""
    import numpy as np
    import workloads as W
    from oracle import attention as OA
    from oracle import quant as Q
    n, t = sample["n"], sample["t"]
    cbk, cbv, cbv2 = sample["cbk"], sample["cbv"], sample["cbv2"]
    Pi, S = sample["Pi"], sample["S"]
    ek = Q.encode_mse(sample["K"], Pi, cbk)
    ev = Q.encode_prod(sample["V"], Pi, S, cbv)
    Q.decode(ek["codes"], ek["norms"], Pi, cbk)
    Q.decode(ev["codes"], ev["norms"], Pi, cbv, ev["signs"], ev["gammas"], S)
    # attention over one slice of the cache: encode the slice (it is the cache state), dequantise,
    # softmax -- the oracle has no code-domain path, so it dequantises the slice
    kk = Q.decode(sample["ck"]["codes"], sample["ck"]["norms"], Pi, cbk)
    vv = Q.decode(sample["cv"]["codes"], sample["cv"]["norms"], Pi, cbv2, sample["cv"]["signs"],
                  sample["cv"]["gammas"], S)
    OA.softmax_attend(sample["q"], kk, vv, 1.0 / math.sqrt(D))
    return 2 * n + 2 * n + 2 * t


def run_reference(args):
    import numpy as np
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import workloads as W
    from oracle import quant as Q
    from oracle.codebook import lloyd_max
    cores = len(os.sched_getaffinity(0))
    n, t = 16384, 65536
    Pi, S = W.rotation(D), W.jl_matrix(D)
    sample = dict(n=n, t=t, Pi=Pi, S=S, cbk=lloyd_max(D, K_BITS), cbv=lloyd_max(D, V_BITS_BLOCK - 1),
                  cbv2=lloyd_max(D, V_BITS_CACHE - 1),
                  K=W.kv_slice(n, D, 3, 20.0, 0.5, 0, W.TAG_K, 0, 0),
                  V=W.kv_slice(n, D, 3, 20.0, 0.5, 0, W.TAG_V, 0, 0),
                  q=W.queries_bf16((ATT_HQ // ATT_HKV, D)))
    ck = W.kv_slice(t, D, 3, 20.0, 0.5, 0, W.TAG_K, 1, 0)
    cv = W.kv_slice(t, D, 3, 20.0, 0.5, 0, W.TAG_V, 1, 0)
    sample["ck"] = Q.encode_mse(ck, Pi, sample["cbk"])
    sample["cv"] = Q.encode_prod(cv, Pi, S, sample["cbv2"])
    for _ in range(args.warmup):
        oracle_step(sample)
    t0 = time.perf_counter()
    units = 0
    for _ in range(args.steps):
        units += oracle_step(sample)
    el = time.perf_counter() - t0
    value = units / el
    desc = (f"per step: Algorithm 1 + 2 encode and decode of {n} K and {n} V vectors (d=128) and the "
            f"dequantise + softmax attention of one KV head slice of {t} tokens for 4 query heads")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * el / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded Gaussian, outlier channels, log-normal norms)",
        "config": workload_config(),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def cpu_baseline_measure(seconds_cap=20.0):
    """The oracle timed on this host on a bounded sample (same units), for the cpu_baseline key."""
    class A:
        steps, warmup, gpus = 1, 0, 1
    import numpy as np
    import workloads as W
    from oracle import quant as Q
    from oracle.codebook import lloyd_max
    n, t = 16384, 65536
    Pi, S = W.rotation(D), W.jl_matrix(D)
    sample = dict(n=n, t=t, Pi=Pi, S=S, cbk=lloyd_max(D, K_BITS), cbv=lloyd_max(D, V_BITS_BLOCK - 1),
                  cbv2=lloyd_max(D, V_BITS_CACHE - 1),
                  K=W.kv_slice(n, D, 3, 20.0, 0.5, 0, W.TAG_K, 0, 0),
                  V=W.kv_slice(n, D, 3, 20.0, 0.5, 0, W.TAG_V, 0, 0),
                  q=W.queries_bf16((ATT_HQ // ATT_HKV, D)))
    sample["ck"] = Q.encode_mse(W.kv_slice(t, D, 3, 20.0, 0.5, 0, W.TAG_K, 1, 0), Pi, sample["cbk"])
    sample["cv"] = Q.encode_prod(W.kv_slice(t, D, 3, 20.0, 0.5, 0, W.TAG_V, 1, 0), Pi, S, sample["cbv2"])
    oracle_step(sample)
    t0 = time.perf_counter()
    units, k = 0, 0
    while True:
        units += oracle_step(sample)
        k += 1
        if time.perf_counter() - t0 > seconds_cap or k >= 10:
            break
    el = time.perf_counter() - t0
    return {"value": units / el, "unit": UNIT, "cores": len(os.sched_getaffinity(0)), "kind": "oracle",
            "sample": f"{k} oracle steps of: encode+decode {n} K and {n} V vectors, attention over one "
                      f"{t}-token KV-head slice (4 query heads); {el:.1f} s"}


def workload_config():
    return {
        "workload": "llama8b_block_encode_decode + decode_attention",
        "encode_block": f"K,V bf16 [{BLK_HEADS}x{BLK_TOKENS}x{D}], K alg1 b={K_BITS}, V alg2 b={V_BITS_BLOCK}",
        "attention": f"B={ATT_B} Hq={ATT_HQ} Hkv={ATT_HKV} d={D} T={ATT_T}, K alg1 b={K_BITS}, "
                     f"V alg2 b={V_BITS_CACHE}, bf16 queries",
        "vectors_per_step": vectors_per_step(),
        "l2": "inputs larger than L2 (packed cache 1.44 GB + 134 MB block per step)",
    }


def vectors_per_step():
    nblk = BLK_HEADS * BLK_TOKENS
    return 2 * nblk + 2 * nblk + 2 * ATT_B * ATT_HKV * ATT_T


# ------------------------------------------------------------------------------------------------
# our arm
# ------------------------------------------------------------------------------------------------

def gen_kv(heads, tokens, d, n_outlier, scale, sigma, seed, device, batch=1):
    """bf16 [batch*heads*tokens, d] following the synthetic recipe (torch generator on device)."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    out = torch.empty((batch * heads, tokens, d), dtype=torch.bfloat16, device=device)
    for h in range(batch * heads):
        x = torch.randn((tokens, d), generator=g, device=device)
        ch = torch.randperm(d, generator=g, device=device)[:n_outlier]
        x[:, ch] *= scale
        if sigma > 0:
            x *= torch.exp(sigma * torch.randn((tokens, 1), generator=g, device=device))
        out[h] = x.to(torch.bfloat16)
    return out.view(-1, d)


def run_ours(args):
    import numpy as np
    import torch
    import torch.distributed as dist
    import kv_cache_vector_encode_b200 as tq
    from kv_cache_vector_encode_b200 import shard
    import workloads as W

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream()

    Pi, S = W.rotation(D), W.jl_matrix(D)
    rot = tq.tq_rotation_prepare(torch.from_numpy(Pi).to(dev), torch.from_numpy(S).to(dev))
    cbk = tq.tq_codebook_init(D, K_BITS)
    cbv = tq.tq_codebook_init(D, V_BITS_BLOCK - 1)
    cbv2 = tq.tq_codebook_init(D, V_BITS_CACHE - 1)

    # the resident packed cache of the attention workload (built once, untimed)
    ncache = ATT_B * ATT_HKV * ATT_T
    kc, kn = tq.empty_mse(ncache, D, K_BITS, dev)
    vc, vs, vn, vg = tq.empty_prod(ncache, D, V_BITS_CACHE, dev)
    per = ATT_HKV * ATT_T
    for b in range(ATT_B):
        kb = gen_kv(ATT_HKV, ATT_T, D, 3, 20.0, 0.5, 1000 + 2 * b + 17 * rank, dev)
        vb = gen_kv(ATT_HKV, ATT_T, D, 3, 20.0, 0.5, 1001 + 2 * b + 17 * rank, dev)
        sl = slice(b * per, (b + 1) * per)
        tq.tq_encode_mse(cbk, kb, rot, kc[sl], kn[sl])
        tq.tq_encode_prod(cbv2, vb, rot, vc[sl], vs[sl], vn[sl], vg[sl])
        del kb, vb
    q = torch.randn((ATT_B, ATT_HQ, D), generator=torch.Generator(device=dev).manual_seed(2 + rank),
                    device=dev).to(torch.bfloat16)
    att_out = torch.empty((ATT_B, ATT_HQ, D), dtype=torch.float32, device=dev)
    ws = torch.empty(tq.tq_attend_workspace_bytes(ATT_B, ATT_HQ, ATT_HKV, ATT_T, D), dtype=torch.uint8, device=dev)
    kn3, vn3 = kn.view(ATT_B, ATT_HKV, ATT_T), vn.view(ATT_B, ATT_HKV, ATT_T)
    vg3 = vg.view(ATT_B, ATT_HKV, ATT_T)

    # the block of each step
    nblk = BLK_HEADS * BLK_TOKENS
    Kb = gen_kv(BLK_HEADS, BLK_TOKENS, D, 3, 20.0, 0.5, 7 + 13 * rank, dev)
    Vb = gen_kv(BLK_HEADS, BLK_TOKENS, D, 3, 20.0, 0.5, 8 + 13 * rank, dev)
    bkc, bkn = tq.empty_mse(nblk, D, K_BITS, dev)
    bvc, bvs, bvn, bvg = tq.empty_prod(nblk, D, V_BITS_BLOCK, dev)
    outk = torch.empty((nblk, D), dtype=torch.float32, device=dev)
    outv = torch.empty((nblk, D), dtype=torch.float32, device=dev)
    tq.tq_sync_check()

    def step(ev=None, bufs=None):
        Kx, Vx, qx, (ckc, ckn, cvc, cvs, cvn, cvg, cout) = bufs or (Kb, Vb, q, (bkc, bkn, bvc, bvs, bvn, bvg, att_out))
        if ev is not None:
            ev[0].record(stream)
        tq.tq_encode_mse(cbk, Kx, rot, ckc, ckn)
        if ev is not None:
            ev[1].record(stream)
        tq.tq_encode_prod(cbv, Vx, rot, cvc, cvs, cvn, cvg)
        if ev is not None:
            ev[2].record(stream)
        tq.tq_decode(cbk, rot, ckc, ckn, outk)
        if ev is not None:
            ev[3].record(stream)
        tq.tq_decode(cbv, rot, cvc, cvn, outv, signs=cvs, gammas=cvg)
        if ev is not None:
            ev[4].record(stream)
        tq.tq_attend_decode(cbk, cbv2, qx, rot, kc, kn3, vc, vn3, cout, v_signs=vs, v_gammas=vg3, ws=ws)
        if ev is not None:
            ev[5].record(stream)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        step()
    tq.tq_sync_check()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(args.steps)]
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    with ClockSampler(torch.cuda.current_device()) as clk:
        e_start.record(stream)
        for k in range(args.steps):
            step(evs[k])
        e_end.record(stream)
        barrier()
    tq.tq_sync_check()
    total_ms = e_start.elapsed_time(e_end)
    parts = {name: statistics.mean(evs[k][i].elapsed_time(evs[k][i + 1]) for k in range(args.steps))
             for i, name in enumerate(["encode_k", "encode_v", "decode_k", "decode_v", "attend"])}
    total_ms = shard.max_over_ranks(total_ms, device=dev)      # device time, max over ranks
    ms_step = total_ms / args.steps
    value = world * vectors_per_step() / (ms_step * 1e-3)

    # end-to-end through the public API with host buffers: inputs from pinned memory each step,
    # results (packed block + attention output) read back
    Kh = Kb.cpu().pin_memory()
    Vh = Vb.cpu().pin_memory()
    qh = q.cpu().pin_memory()
    res = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in (bkc, bkn, bvc, bvs, bvn, bvg, att_out)]
    h2d = Kh.numel() * 2 + Vh.numel() * 2 + qh.numel() * 2
    d2h = sum(r.numel() * r.element_size() for r in res)

    # Two buffer sets: the inputs of step k+1 are copied in (one copy stream) while step k computes,
    # and the results of step k are copied out (a second copy stream) while step k+1 computes.
    # Every step's copies lie inside the timed region, which ends when the last results are home.
    sets = [(Kb, Vb, q, (bkc, bkn, bvc, bvs, bvn, bvg, att_out))]
    sets.append((torch.empty_like(Kb), torch.empty_like(Vb), torch.empty_like(q),
                 tuple(torch.empty_like(t) for t in (bkc, bkn, bvc, bvs, bvn, bvg, att_out))))
    h2d_s, d2h_s = torch.cuda.Stream(), torch.cuda.Stream()

    def e2e_run(n, start=None, end=None):
        ev_in = [torch.cuda.Event() for _ in range(2)]      # inputs of the set are on the device
        ev_done = [torch.cuda.Event() for _ in range(2)]    # the step using the set has finished
        ev_out = [torch.cuda.Event() for _ in range(2)]     # the set's results are home
        if start is not None:
            start.record(h2d_s)

        def copy_in(k):
            Kx, Vx, qx, _ = sets[k % 2]
            with torch.cuda.stream(h2d_s):
                if k >= 2:
                    h2d_s.wait_event(ev_done[k % 2])           # step k-2 has read this set
                Kx.copy_(Kh, non_blocking=True)
                Vx.copy_(Vh, non_blocking=True)
                qx.copy_(qh, non_blocking=True)
                ev_in[k % 2].record(h2d_s)

        copy_in(0)
        for k in range(n):
            if k + 1 < n:
                copy_in(k + 1)
            stream.wait_event(ev_in[k % 2])
            if k >= 2:
                stream.wait_event(ev_out[k % 2])               # results of step k-2 are home
            step(bufs=sets[k % 2])
            ev_done[k % 2].record(stream)
            with torch.cuda.stream(d2h_s):
                d2h_s.wait_event(ev_done[k % 2])
                for r, t in zip(res, sets[k % 2][3]):
                    r.copy_(t, non_blocking=True)
                ev_out[k % 2].record(d2h_s)
        if end is not None:
            d2h_s.wait_stream(h2d_s)
            end.record(d2h_s)

    e2e_run(2)
    barrier()
    a, b2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_steps = max(3, min(args.steps, 10))
    e2e_run(e2e_steps, a, b2)
    barrier()
    e2e_ms = a.elapsed_time(b2) / e2e_steps
    e2e_ms = shard.max_over_ranks(e2e_ms, device=dev)
    e2e_value = world * vectors_per_step() / (e2e_ms * 1e-3)

    peak, peak_kind = peaks()
    att_bytes = B_ATT_TOKEN_HEAD * ATT_B * ATT_HKV * ATT_T + ATT_B * ATT_HQ * D * (2 + 4)
    att_gbs = att_bytes / (parts["attend"] * 1e-3) / 1e9
    traffic = None
    prof = os.path.join(ROOT, "profiles", "attend_main_decode_attention_traffic.json")
    if os.path.exists(prof):
        try:
            traffic = json.load(open(prof)).get("dram_bytes_per_launch")
        except Exception:
            traffic = None
    comp_bytes = {
        "encode_k": B_ENC_K * nblk, "encode_v": B_ENC_V * nblk,
        "decode_k": B_DEC_K * nblk, "decode_v": B_DEC_V * nblk, "attend": att_bytes,
    }
    breakdown = {}
    for name, ms in parts.items():
        gbs = comp_bytes[name] / (ms * 1e-3) / 1e9
        breakdown[name] = {"ms": round(ms, 4), "GB/s": round(gbs, 1), "frac_hbm": round(gbs / peak, 4)}
    breakdown["encode_vectors_per_s"] = 2 * nblk / ((parts["encode_k"] + parts["encode_v"]) * 1e-3)
    breakdown["attention_kv_tokens_per_s"] = ATT_B * ATT_T / (parts["attend"] * 1e-3)
    breakdown["attention_query_tokens_per_s"] = ATT_B / (parts["attend"] * 1e-3)
    step_bytes = sum(comp_bytes.values())
    breakdown["step_frac_hbm"] = round(step_bytes / (ms_step * 1e-3) / 1e9 / peak, 4)

    if rank == 0:
        cpu = cpu_baseline_measure() if (world == 1 and not args.no_cpu_baseline) else None
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16 in; int8/fp16 tensor-core products, fp32 accumulate",
            "data": "synthetic (seeded Gaussian, outlier channels x20, log-normal token norms); no datasets",
            "config": workload_config(),
            "roofline": {"bound": "hbm", "kernel": "tq_attend_decode (prep + main + combine)",
                         "achieved": round(att_gbs, 1), "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                         "frac": round(att_gbs / peak, 4), "traffic": traffic,
                         "algorithmic_bytes_per_launch": att_bytes},
            "breakdown": breakdown,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": e2e_ms},
            "gpu_launches": args.steps * 7,
            "clocks": clk.summary(),
        }
        if cpu is not None:
            line["cpu_baseline"] = cpu
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_only_block(args):
    """Times the block kernels alone (encode K, encode V, decode K, decode V) on the llama8b block shape
    (a profiling entry point; prints one JSON line with the mean time of each call)."""
    import torch
    import kv_cache_vector_encode_b200 as tq
    import workloads as W
    dev = torch.device("cuda")
    Pi, S = W.rotation(D), W.jl_matrix(D)
    rot = tq.tq_rotation_prepare(torch.from_numpy(Pi).to(dev), torch.from_numpy(S).to(dev))
    cbk, cbv = tq.tq_codebook_init(D, K_BITS), tq.tq_codebook_init(D, V_BITS_BLOCK - 1)
    nblk = BLK_HEADS * BLK_TOKENS
    Kb = gen_kv(BLK_HEADS, BLK_TOKENS, D, 3, 20.0, 0.5, 7, dev)
    Vb = gen_kv(BLK_HEADS, BLK_TOKENS, D, 3, 20.0, 0.5, 8, dev)
    kc, kn = tq.empty_mse(nblk, D, K_BITS, dev)
    vc, vs, vn, vg = tq.empty_prod(nblk, D, V_BITS_BLOCK, dev)
    outk = torch.empty((nblk, D), dtype=torch.float32, device=dev)
    outv = torch.empty((nblk, D), dtype=torch.float32, device=dev)
    calls = {"encode_k": lambda: tq.tq_encode_mse(cbk, Kb, rot, kc, kn),
             "encode_v": lambda: tq.tq_encode_prod(cbv, Vb, rot, vc, vs, vn, vg),
             "decode_k": lambda: tq.tq_decode(cbk, rot, kc, kn, outk),
             "decode_v": lambda: tq.tq_decode(cbv, rot, vc, vn, outv, signs=vs, gammas=vg)}
    res = {}
    for name, f in calls.items():
        for _ in range(args.warmup):
            f()
        torch.cuda.synchronize()
        a, b2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(args.steps):
            f()
        b2.record()
        torch.cuda.synchronize()
        res[name + "_us"] = a.elapsed_time(b2) / args.steps * 1e3
    tq.tq_sync_check()
    print(json.dumps({"only": "block", "vectors": nblk, **res}), flush=True)
    return 0


def run_only_attend(args):
    """Times tq_attend_decode alone on the decode-attention shape with `--att-tokens` cached tokens
    (a profiling entry point; prints one JSON line with the mean time of a call)."""
    import torch
    import kv_cache_vector_encode_b200 as tq
    import workloads as W
    dev = torch.device("cuda")
    T = args.att_tokens
    Pi, S = W.rotation(D), W.jl_matrix(D)
    rot = tq.tq_rotation_prepare(torch.from_numpy(Pi).to(dev), torch.from_numpy(S).to(dev))
    cbk, cbv2 = tq.tq_codebook_init(D, K_BITS), tq.tq_codebook_init(D, V_BITS_CACHE - 1)
    n = ATT_B * ATT_HKV * T
    kc, kn = tq.empty_mse(n, D, K_BITS, dev)
    vc, vs, vn, vg = tq.empty_prod(n, D, V_BITS_CACHE, dev)
    per = ATT_HKV * T
    for b in range(ATT_B):
        sl = slice(b * per, (b + 1) * per)
        tq.tq_encode_mse(cbk, gen_kv(ATT_HKV, T, D, 3, 20.0, 0.5, 1000 + 2 * b, dev), rot, kc[sl], kn[sl])
        tq.tq_encode_prod(cbv2, gen_kv(ATT_HKV, T, D, 3, 20.0, 0.5, 1001 + 2 * b, dev), rot, vc[sl], vs[sl], vn[sl],
                          vg[sl])
    q = torch.randn((ATT_B, ATT_HQ, D), generator=torch.Generator(device=dev).manual_seed(2), device=dev)
    q = q.to(torch.bfloat16)
    out = torch.empty((ATT_B, ATT_HQ, D), dtype=torch.float32, device=dev)
    ws = torch.empty(tq.tq_attend_workspace_bytes(ATT_B, ATT_HQ, ATT_HKV, T, D), dtype=torch.uint8, device=dev)
    kn3, vn3, vg3 = kn.view(ATT_B, ATT_HKV, T), vn.view(ATT_B, ATT_HKV, T), vg.view(ATT_B, ATT_HKV, T)

    def call():
        tq.tq_attend_decode(cbk, cbv2, q, rot, kc, kn3, vc, vn3, out, v_signs=vs, v_gammas=vg3, ws=ws)

    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()
    a, b2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(args.steps):
        call()
    b2.record()
    torch.cuda.synchronize()
    tq.tq_sync_check()
    ms = a.elapsed_time(b2) / args.steps
    byts = B_ATT_TOKEN_HEAD * ATT_B * ATT_HKV * T
    print(json.dumps({"only": "attend", "tokens": T, "us_per_call": ms * 1e3, "GB/s": byts / (ms * 1e-3) / 1e9}),
          flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--only", choices=["attend", "block"], default=None,
                    help="profiling entry point: time one path alone (not a bench line)")
    ap.add_argument("--att-tokens", type=int, default=ATT_T)
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    if args.only == "attend":
        return run_only_attend(args)
    if args.only == "block":
        return run_only_block(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
