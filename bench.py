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


TRAFFIC_SOURCES = ("attend.cu", "sm100.cuh")


def traffic_from_record(rec, sources):
    """DRAM bytes per launch from an ncu capture record, or None unless the sha256 recorded in it
    equals the sha256 of `sources` (the kernel's source files' bytes, in order): a figure taken on
    an earlier version of the kernel is not reported."""
    import hashlib
    h = hashlib.sha256()
    for b in sources:
        h.update(b)
    if not isinstance(rec, dict) or rec.get("source_sha256") != h.hexdigest():
        return None
    return rec.get("dram_bytes_per_launch")


def captured_traffic():
    """DRAM bytes of one attention launch from the committed capture (profiles/), or None."""
    prof = os.path.join(ROOT, "profiles", "attend_main_decode_attention_traffic.json")
    try:
        rec = json.load(open(prof))
        srcs = []
        for src in TRAFFIC_SOURCES:
            with open(os.path.join(ROOT, "kv_cache_vector_encode_b200", "csrc", src), "rb") as f:
                srcs.append(f.read())
        return traffic_from_record(rec, srcs)
    except Exception:
        return None


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def tensor_peak():
    """Dense fp16 / bf16 tensor peak (TFLOP/s): the measured burst figure, else the fallback."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        return 1590.0, "fallback"


_CLOCK_CHILD = r"""
import select, sys
import pynvml as nv
nv.nvmlInit()
key, period = sys.argv[1], float(sys.argv[2])
try:
    h = nv.nvmlDeviceGetHandleByUUID(key)
except Exception:
    h = nv.nvmlDeviceGetHandleByIndex(int(sys.argv[3]))
mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
bits = [nv.nvmlClocksEventReasonHwSlowdown, nv.nvmlClocksEventReasonHwThermalSlowdown,
        nv.nvmlClocksEventReasonSwThermalSlowdown, nv.nvmlClocksEventReasonSwPowerCap]
out = []
print("ready", flush=True)
while True:
    try:
        sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
        r = int(nv.nvmlDeviceGetCurrentClocksEventReasons(h))
        out.append("%d,%d,%s" % (sm, mx, ",".join("1" if r & b else "0" for b in bits)))
    except Exception:
        pass
    if select.select([sys.stdin], [], [], period)[0]:
        break                                   # the parent closed our stdin: the region is over
print("\n".join(out), flush=True)
"""


class ClockSampler:
    """SM clock and throttle-reason samples while the timed region runs. A child process polls NVML
    every 2 ms (a thread of this process would compete for the interpreter lock with the launch
    loop), else nvidia-smi reports every 20 ms. Reads settings only."""

    SMI_FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                  "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, index: int, period_s: float = 0.002):
        self.index = index
        self.period = period_s
        self.proc = None
        self.thread = None
        self.samples = []          # (sm_mhz, max_mhz, set of reason names)
        self.source = None

    def _parse(self, line):
        parts = [x.strip() for x in line.strip().split(",")]
        if len(parts) < 6:
            return
        try:
            sm, mx = float(parts[0]), float(parts[1])
        except ValueError:
            return
        act = [v.lower().startswith("active") or v == "1" for v in parts[2:6]]
        self.samples.append((sm, mx, {nm for nm, a in zip(self.NAMES, act) if a}))

    def _start_nvml_child(self):
        import torch
        uuid = str(torch.cuda.get_device_properties(self.index).uuid)
        uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        proc = subprocess.Popen([sys.executable, "-c", _CLOCK_CHILD, uuid, str(self.period), str(self.index)],
                                stdin=subprocess.PIPE, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        if proc.stdout.readline().strip() != "ready":
            proc.kill()
            proc.wait()
            raise RuntimeError("NVML sampler did not start")
        return proc

    def __enter__(self):
        try:
            self.proc = self._start_nvml_child()
            self.source = "nvml in a child process, every 2 ms"
        except Exception:
            try:
                self.proc = subprocess.Popen(
                    ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.SMI_FIELDS}",
                     "--format=csv,noheader,nounits", "-lms", "20"],
                    stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
                self.thread = threading.Thread(target=lambda: [self._parse(ln) for ln in self.proc.stdout],
                                               daemon=True)
                self.thread.start()
                self.source = "nvidia-smi, every 20 ms"
            except Exception:
                self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is None:
            return
        if self.thread is None:
            # the NVML child: closing its stdin ends the loop, then it prints its samples
            try:
                out, _ = self.proc.communicate(input="", timeout=30)
                for ln in out.splitlines():
                    self._parse(ln)
            except Exception:
                self.proc.kill()
                self.proc.wait()
            return
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.thread.join(timeout=5)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "source": self.source}
        sm = [x[0] for x in self.samples]
        reasons = set().union(*[x[2] for x in self.samples])
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(x[1] for x in self.samples),
                "sm_mhz_min": min(sm), "reasons": sorted(reasons), "samples": len(sm), "source": self.source}


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
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": desc,
                         "other_workloads": oracle_per_workload()},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def oracle_per_workload():
    """The oracle on bounded samples of each workload (host cores; vectors or pairs per second)."""
    import numpy as np
    import workloads as W
    from oracle import attention as OA
    from oracle import quant as Q
    from oracle.codebook import lloyd_max
    res = {}

    def clock(fn):
        t0 = time.perf_counter()
        fn()
        return time.perf_counter() - t0

    # tiny: 4096 x 128 fp32, Algorithm 1 encode + decode at b = 1..4 (the whole set)
    d = 128
    Pi = W.rotation(d)
    x = W.gaussian(4096, d)
    cbs = {b: lloyd_max(d, b) for b in (1, 2, 3, 4)}

    def tiny():
        for b, cb in cbs.items():
            e = Q.encode_mse(x, Pi, cb)
            Q.decode(e["codes"], e["norms"], Pi, cb)
    el = clock(tiny)
    res["tiny_4096x128_f32"] = {"vectors_per_s": 4 * 2 * 4096 / el, "sample": "whole set, b = 1..4", "s": el}
    # TinyLlama-shaped block at d = 64: a 4096-token head of K (Algorithm 1 b=3) and of V (Algorithm 2 b=2)
    d = 64
    Pi, S = W.rotation(d), W.jl_matrix(d)
    K = W.kv_slice(4096, d, 4, 20.0, 0.0, 0, W.TAG_K, 0, 0)
    V = W.kv_slice(4096, d, 4, 20.0, 0.0, 0, W.TAG_V, 0, 0)
    cbk, cbv = lloyd_max(d, 3), lloyd_max(d, 1)

    def tl():
        ek = Q.encode_mse(K, Pi, cbk)
        ev = Q.encode_prod(V, Pi, S, cbv)
        Q.decode(ek["codes"], ek["norms"], Pi, cbk)
        Q.decode(ev["codes"], ev["norms"], Pi, cbv, ev["signs"], ev["gammas"], S)
    el = clock(tl)
    res["tinyllama_block_32x4096x64"] = {"vectors_per_s": 4 * 4096 / el,
                                         "sample": "one head: 4096 K and 4096 V encoded and decoded", "s": el}
    # vector search at d = 1536: 2048 database vectors encoded (Algorithm 2 b=4), 64 queries scored
    d = 1536
    Pi, S = W.rotation(d), W.jl_matrix(d)
    X = W.unit_rows(2048, d)
    qs = W.unit_rows(64, d, tag=W.TAG_Q)
    cb3 = lloyd_max(d, 3)
    st = {}

    def enc():
        st["e"] = Q.encode_prod(X, Pi, S, cb3)
    el_e = clock(enc)

    def scan():
        e = st["e"]
        xh = Q.decode(e["codes"], e["norms"], Pi, cb3, e["signs"], e["gammas"], S)
        OA.topk(OA.scores(qs, xh), 10)
    el_s = clock(scan)
    res["vector_search_1e6x1536"] = {"encode_vectors_per_s": 2048 / el_e, "score_pairs_per_s": 64 * 2048 / el_s,
                                     "sample": "2048 database vectors, 64 queries", "s": el_e + el_s}
    return res


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
    per = oracle_per_workload()
    return {"value": units / el, "unit": UNIT, "cores": len(os.sched_getaffinity(0)), "kind": "oracle",
            "other_workloads": per,
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
        Kx, Vx, qx, (ckc, ckn, cvc, cvs, cvn, cvg, cout, cok, cov) = bufs or (
            Kb, Vb, q, (bkc, bkn, bvc, bvs, bvn, bvg, att_out, outk, outv))
        if ev is not None:
            ev[0].record(stream)
        tq.tq_encode_mse(cbk, Kx, rot, ckc, ckn)
        if ev is not None:
            ev[1].record(stream)
        tq.tq_encode_prod(cbv, Vx, rot, cvc, cvs, cvn, cvg)
        if ev is not None:
            ev[2].record(stream)
        tq.tq_decode(cbk, rot, ckc, ckn, cok)
        if ev is not None:
            ev[3].record(stream)
        tq.tq_decode(cbv, rot, cvc, cvn, cov, signs=cvs, gammas=cvg)
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
    # every result of the step read back (packed block, both decoded blocks, attention output)
    Kh = Kb.cpu().pin_memory()
    Vh = Vb.cpu().pin_memory()
    qh = q.cpu().pin_memory()
    outs = (bkc, bkn, bvc, bvs, bvn, bvg, att_out, outk, outv)
    res = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in outs]
    h2d = Kh.numel() * 2 + Vh.numel() * 2 + qh.numel() * 2
    d2h = sum(r.numel() * r.element_size() for r in res)

    # Two buffer sets: the inputs of step k+1 are copied in (one copy stream) while step k computes,
    # and the results of step k are copied out (a second copy stream) while step k+1 computes.
    # Every step's copies lie inside the timed region, which ends when the last results are home.
    sets = [(Kb, Vb, q, outs)]
    sets.append((torch.empty_like(Kb), torch.empty_like(Vb), torch.empty_like(q),
                 tuple(torch.empty_like(t) for t in outs)))
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
    traffic = captured_traffic()
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

    extra = None
    if rank == 0 and not args.no_extra:
        extra = extra_workloads(dev, peak, tensor_peak()[0])
    if world > 1:
        dist.barrier()
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
            "other_workloads": extra,
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


def _timed(fn, iters, warmup=3):
    """Mean device time (ms) of fn() over `iters` calls on the current stream (CUDA events)."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(iters):
        fn()
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / iters


def _graph_timed(fn, reps, iters=20):
    """Mean device time (ms) of fn() when `reps` calls are captured in one CUDA graph and the graph is
    replayed `iters` times (removes host launch overhead for the small workloads); None if the calls
    cannot be captured."""
    import torch
    try:
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            fn()
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(reps):
                fn()
        g.replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(iters):
            g.replay()
        b.record()
        torch.cuda.synchronize()
        ms = a.elapsed_time(b) / (iters * reps)
        del g
        return ms
    except Exception:
        torch.cuda.synchronize()
        return None


def extra_workloads(dev, peak_hbm, peak_tensor):
    """The other workloads measured beside the step (each call timed alone with CUDA events; not part
    of the step's value): the tiny correctness set (4096 x 128 fp32, Algorithm 1 at b = 1..4), the
    TinyLlama-shaped block (K, V bf16 [32 x 4096 x 64], K Algorithm 1 b=3, V Algorithm 2 b=2) and
    the vector-search scan (1e6 x 1536 fp32 unit rows, Algorithm 2 b=4, 1024 queries, top-10)."""
    import torch
    import kv_cache_vector_encode_b200 as tq
    import workloads as W
    out = {}
    # -- tiny: 4096 x 128 fp32, Algorithm 1 encode + decode at b = 1..4 (launch-bound)
    d, n = 128, 4096
    Pi, S = W.rotation(d), W.jl_matrix(d)
    rot = tq.tq_rotation_prepare(torch.from_numpy(Pi).to(dev), torch.from_numpy(S).to(dev))
    x = torch.randn((n, d), generator=torch.Generator(device=dev).manual_seed(0), device=dev)
    xd = torch.empty((n, d), dtype=torch.float32, device=dev)
    tiny = {}
    for b in (1, 2, 3, 4):
        cb = tq.tq_codebook_init(d, b)
        c, nn = tq.empty_mse(n, d, b, dev)
        enc = lambda: tq.tq_encode_mse(cb, x, rot, c, nn)
        dec = lambda: tq.tq_decode(cb, rot, c, nn, xd)
        both = lambda: (enc(), dec())
        ms = _timed(both, 50)
        msg = _graph_timed(both, 50)
        tiny[f"b{b}"] = {"encode_decode_ms": round(ms, 5), "vectors_per_s": 2 * n / (ms * 1e-3),
                         "graph_ms": None if msg is None else round(msg, 5),
                         "graph_vectors_per_s": None if msg is None else 2 * n / (msg * 1e-3)}
    out["tiny_4096x128_f32"] = tiny
    # -- TinyLlama-shaped block: K, V bf16 [32 x 4096 x 64]
    d, heads, tokens = 64, 32, 4096
    n = heads * tokens
    Pi, S = W.rotation(d), W.jl_matrix(d)
    rot64 = tq.tq_rotation_prepare(torch.from_numpy(Pi).to(dev), torch.from_numpy(S).to(dev))
    K = W.kv_slices_device(heads, tokens, d, 4, 20.0, 0.0, 31, dev)
    V = W.kv_slices_device(heads, tokens, d, 4, 20.0, 0.0, 32, dev)
    cbk, cbv = tq.tq_codebook_init(d, 3), tq.tq_codebook_init(d, 1)
    kc, kn = tq.empty_mse(n, d, 3, dev)
    vc, vs, vn, vg = tq.empty_prod(n, d, 2, dev)
    kd = torch.empty((n, d), dtype=torch.float32, device=dev)
    vd = torch.empty((n, d), dtype=torch.float32, device=dev)
    calls = {"encode_k": (lambda: tq.tq_encode_mse(cbk, K, rot64, kc, kn), 2 * d + 3 * d // 8 + 2),
             "encode_v": (lambda: tq.tq_encode_prod(cbv, V, rot64, vc, vs, vn, vg), 2 * d + d // 8 + d // 8 + 4),
             "decode_k": (lambda: tq.tq_decode(cbk, rot64, kc, kn, kd), 3 * d // 8 + 2 + 4 * d),
             "decode_v": (lambda: tq.tq_decode(cbv, rot64, vc, vn, vd, signs=vs, gammas=vg), d // 8 + d // 8 + 4 + 4 * d)}
    blk = {}
    for name, (fn, bpv) in calls.items():
        ms = _timed(fn, 50)
        msg = _graph_timed(fn, 20)
        best = min(ms, msg) if msg is not None else ms
        gbs = bpv * n / (best * 1e-3) / 1e9
        blk[name] = {"ms": round(ms, 5), "graph_ms": None if msg is None else round(msg, 5),
                     "vectors_per_s": n / (best * 1e-3), "GB/s": round(gbs, 1), "frac_hbm": round(gbs / peak_hbm, 4)}
    out["tinyllama_block_32x4096x64"] = blk
    del K, V, kc, kn, vc, vs, vn, vg, kd, vd
    # -- mixed widths per channel group: the llama8b-shaped K block at widths (3, 3, 2, 2) = 2.5 bits
    d = 128
    nblk = BLK_HEADS * BLK_TOKENS
    Pi, S = W.rotation(d), W.jl_matrix(d)
    rotm = tq.tq_rotation_prepare(torch.from_numpy(Pi).to(dev), torch.from_numpy(S).to(dev))
    gb = [3, 3, 2, 2]
    Km = W.kv_slices_device(BLK_HEADS, BLK_TOKENS, d, 3, 20.0, 0.5, 51, dev)
    cm = torch.empty((nblk, sum(gb)), dtype=torch.int32, device=dev)
    nm = torch.empty((nblk,), dtype=torch.float16, device=dev)
    xm = torch.empty((nblk, d), dtype=torch.float32, device=dev)
    ms_me = _timed(lambda: tq.tq_encode_mse_mixed(gb, Km, rotm, cm, nm), 20)
    ms_md = _timed(lambda: tq.tq_decode_mixed(gb, rotm, cm, nm, xm), 20)
    be = nblk * (2 * d + 4 * sum(gb) + 2)
    bd = nblk * (4 * sum(gb) + 2 + 4 * d)
    out["mixed_widths_3322_llama8b_k_block"] = {
        "bits_per_coordinate": sum(gb) * 32 / d,
        "encode_ms": round(ms_me, 4), "encode_GB/s": round(be / (ms_me * 1e-3) / 1e9, 1),
        "encode_frac_hbm": round(be / (ms_me * 1e-3) / 1e9 / peak_hbm, 4),
        "decode_ms": round(ms_md, 4), "decode_GB/s": round(bd / (ms_md * 1e-3) / 1e9, 1),
        "decode_frac_hbm": round(bd / (ms_md * 1e-3) / 1e9 / peak_hbm, 4)}
    del Km, cm, nm, xm
    # -- prefill: 128 new query tokens at the end of a 32768-token cache, batch 1, 32 / 8 heads
    Bp, Hqp, Hkvp, Tp, Qn = 1, 32, 8, 32768, 128
    cbk, cbv = tq.tq_codebook_init(d, 3), tq.tq_codebook_init(d, 1)
    npf = Bp * Hkvp * Tp
    pkc, pkn = tq.empty_mse(npf, d, 3, dev)
    pvc, pvs, pvn, pvg = tq.empty_prod(npf, d, 2, dev)
    tq.tq_encode_mse(cbk, W.kv_slices_device(Hkvp, Tp, d, 3, 20.0, 0.5, 61, dev), rotm, pkc, pkn)
    tq.tq_encode_prod(cbv, W.kv_slices_device(Hkvp, Tp, d, 3, 20.0, 0.5, 62, dev), rotm, pvc, pvs, pvn, pvg)
    qp = torch.randn((Bp, Qn, Hqp, d), generator=torch.Generator(device=dev).manual_seed(63), device=dev).to(torch.bfloat16)
    op = torch.empty((Bp, Qn, Hqp, d), dtype=torch.float32, device=dev)
    wsp = torch.empty(tq.tq_attend_prefill_workspace_bytes(Bp, Hqp, Hkvp, Qn, Tp, d), dtype=torch.uint8, device=dev)
    sh = (Bp, Hkvp, Tp)
    ms_pf = _timed(lambda: tq.tq_attend_prefill(cbk, cbv, qp, rotm, pkc, pkn.view(sh), pvc, pvn.view(sh), op,
                                                 v_signs=pvs, v_gammas=pvg.view(sh), ws=wsp), 5)
    qpass = max(1, 8 // (Hqp // Hkvp))
    passes = -(-Qn // qpass)
    streamed = sum(B_ATT_TOKEN_HEAD * Bp * Hkvp * (Tp - Qn + j0 + min(qpass, Qn - j0)) for j0 in range(0, Qn, qpass))
    flops = sum(2 * 2 * d * Hqp * (Tp - Qn + j + 1) for j in range(Qn)) * Bp       # q.k and p.v per visible token
    out["prefill_B1_32x8_T32768_Q128"] = {
        "ms": round(ms_pf, 3), "query_tokens_per_s": Bp * Qn / (ms_pf * 1e-3), "passes": passes,
        "cache_bytes_streamed_GB": round(streamed / 1e9, 3),
        "frac_hbm": round(streamed / (ms_pf * 1e-3) / 1e9 / peak_hbm, 4),
        "frac_tensor_algorithmic": round(flops / (ms_pf * 1e-3) / 1e12 / peak_tensor, 5)}
    del pkc, pkn, pvc, pvs, pvn, pvg, wsp
    # -- vector search: 1e6 x 1536 fp32 unit rows, Algorithm 2 at b = 4, 1024 queries, top-10
    d, n, nq, k = 1536, 1_000_000, 1024, 10
    Pi, S = W.rotation(d), W.jl_matrix(d)
    rotv = tq.tq_rotation_prepare(torch.from_numpy(Pi).to(dev), torch.from_numpy(S).to(dev))
    g = torch.Generator(device=dev).manual_seed(41)
    X = torch.empty((n, d), dtype=torch.float32, device=dev)
    for r0 in range(0, n, 100_000):
        blkx = torch.randn((min(100_000, n - r0), d), generator=g, device=dev)
        X[r0:r0 + blkx.shape[0]] = blkx / blkx.norm(dim=1, keepdim=True)
    qv = torch.randn((nq, d), generator=g, device=dev)
    qv = qv / qv.norm(dim=1, keepdim=True)
    cb3 = tq.tq_codebook_init(d, 3)
    c, sg, nn, gm = tq.empty_prod(n, d, 4, dev)
    ws = torch.empty(max(16, tq.tq_encode_workspace_bytes(n, d, 2)), dtype=torch.uint8, device=dev)
    ms_enc = _timed(lambda: tq.tq_encode_prod(cb3, X, rotv, c, sg, nn, gm, ws=ws), 3)
    ids = torch.empty((nq, k), dtype=torch.int32, device=dev)
    sc = torch.empty((nq, k), dtype=torch.float32, device=dev)
    wss = torch.empty(max(16, tq.tq_scores_workspace_bytes(nq, n, d, k)), dtype=torch.uint8, device=dev)
    ms_sc = _timed(lambda: tq.tq_scores(cb3, qv, rotv, c, nn, signs=sg, gammas=gm, k=k, topk_ids=ids,
                                        topk_scores=sc, ws=wss), 3)
    tq.tq_sync_check()
    # algorithmic flops: encode 2 d^2 (Pi x) + 2 d^2 (T rho) per vector; scores 2 d (<q', c>) + 2 d
    # (<q'', z>) per (query, vector). Issued: the tiled encoder's split products (2 or 3 for Pi x with
    # bf16 / fp32 input: 3 here; 3 for T rho); the scores GEMM's K = (Walsh planes + sign plane) d
    # against two fp16 query parts.
    enc_alg = 4.0 * d * d * n
    enc_iss = 2.0 * d * d * (3 + 3) * n
    mk = 4                                   # Walsh planes of a 3-bit codebook
    sc_alg = 4.0 * d * n * nq
    sc_iss = 2.0 * (mk + 1) * d * 2 * n * nq
    enc_bytes = n * (4 * d + 2 * d // 8 + d // 8 + 4 + d // 8)
    out["vector_search_1e6x1536"] = {
        "encode_ms": round(ms_enc, 3), "encode_vectors_per_s": n / (ms_enc * 1e-3),
        "encode_frac_tensor_algorithmic": round(enc_alg / (ms_enc * 1e-3) / 1e12 / peak_tensor, 4),
        "encode_frac_tensor_issued": round(enc_iss / (ms_enc * 1e-3) / 1e12 / peak_tensor, 4),
        "encode_frac_hbm": round(enc_bytes / (ms_enc * 1e-3) / 1e9 / peak_hbm, 4),
        "scores_topk_ms": round(ms_sc, 3),
        "scores_frac_tensor_algorithmic": round(sc_alg / (ms_sc * 1e-3) / 1e12 / peak_tensor, 4),
        "scores_frac_tensor_issued": round(sc_iss / (ms_sc * 1e-3) / 1e12 / peak_tensor, 4),
        "scores_frac_hbm": round(n * (3 * d // 8 + d // 8 + 4) / (ms_sc * 1e-3) / 1e9 / peak_hbm, 4),
        "peak_tensor_tflops": peak_tensor,
    }
    del X, c, sg, nn, gm, ws, wss
    torch.cuda.empty_cache()
    return out


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


def run_only_tiled(args):
    """Times tq_encode_prod on `--tiled-n` unit-norm fp32 rows of d = 1536 at 4 bits (the vector-search
    encode, the tiled kernel and its gamma fix-up; a profiling entry point, not a bench line)."""
    import torch
    import kv_cache_vector_encode_b200 as tq
    import workloads as W
    dev = torch.device("cuda")
    d, n = 1536, args.tiled_n
    Pi, S = W.rotation(d), W.jl_matrix(d)
    rot = tq.tq_rotation_prepare(torch.from_numpy(Pi).to(dev), torch.from_numpy(S).to(dev))
    g = torch.Generator(device=dev).manual_seed(41)
    X = torch.randn((n, d), generator=g, device=dev)
    X = X / X.norm(dim=1, keepdim=True)
    cb = tq.tq_codebook_init(d, 3)
    c, sg, nn, gm = tq.empty_prod(n, d, 4, dev)
    ws = torch.empty(max(16, tq.tq_encode_workspace_bytes(n, d, 2)), dtype=torch.uint8, device=dev)
    ms = _timed(lambda: tq.tq_encode_prod(cb, X, rot, c, sg, nn, gm, ws=ws), args.steps, warmup=args.warmup)
    tq.tq_sync_check()
    print(json.dumps({"only": "tiled", "n": n, "d": d, "ms_per_call": ms, "vectors_per_s": n / (ms * 1e-3)}), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true", help="skip the other workloads' measurements")
    ap.add_argument("--only", choices=["attend", "block", "tiled"], default=None,
                    help="profiling entry point: time one path alone (not a bench line)")
    ap.add_argument("--att-tokens", type=int, default=ATT_T)
    ap.add_argument("--tiled-n", type=int, default=16384)
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    if args.only == "attend":
        return run_only_attend(args)
    if args.only == "block":
        return run_only_block(args)
    if args.only == "tiled":
        return run_only_tiled(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
