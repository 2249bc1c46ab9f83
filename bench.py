#!/usr/bin/env python
"""Benchmark of the blockwise bit-codebook hot path on B200.

One step = one pass of every operation of the path over one batch of resident
synthetic input (default workload "c5", the large streaming case):
    16384 x 16384 bf16 weight ~ N(0, 0.02), seed 7
      kbit_quantize   K=3 -> kbit_dequantize K=3 (bf16 out)
      kbit_quantize   K=5 -> kbit_dequantize K=5 (bf16 out)
      dequantize_4bit_nested NF4 (16-entry normal-float table), outer blocksize 64,
      inner blocksize 256, bf16 out, same element count.
Every input is larger than the 126 MB L2, so no flush is needed between steps.

Metric: achieved HBM GB/s (algorithmic bytes / time) for the whole step, plus
per kernel GB/s, Gelem/s and the fraction of the measured HBM copy bandwidth.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {bbc,reference}]

N > 1 runs under torchrun, one rank per GPU, each rank on its own full copy of
the workload (weak scaling; the path needs no collective). The reference arm
(--impl reference) times the CPU oracle on a bounded sample of the workload.
"""
import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "achieved HBM GB/s and Gelem/s per kernel; fraction of B200 HBM roofline"
FALLBACK_HBM_GBS = 6650.0


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["bbc", "reference"], default="bbc")
    ap.add_argument("--workload", choices=["c5"], default="c5")
    ap.add_argument("--n", type=int, default=None,
                    help="override the element count (profiling of a smaller case)")
    ap.add_argument("--ops", default=None,
                    help="comma-separated subset of quantize_k3,dequantize_k3,quantize_k5,"
                         "dequantize_k5,nested_nf4_bs64, {quantize,dequantize}_k{2,4}, or the E4M4-absmax ops "
                         "{quantize,dequantize}_k{3,4,5}_e4m4, or quantize_4bit_nf4_bs{64,32}, "
                         "quantize_nested_nf4_bs{64,32} (profiling)")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the c1-c4 cells that the default 1-GPU line carries in per_config")
    ap.add_argument("--linear-case", default=None, metavar="FMT:M[:N:K]",
                    help="profiling case: build one fused-linear weight (FMT nested or kbit4, bf16 "
                         "activations, N = K = 4096 unless given) and call the entry point 4 times")
    ap.add_argument("--linear-shapes", default=None, metavar="M,M,...",
                    help="with --linear: only the control shapes with these activation counts")
    ap.add_argument("--linear", action="store_true",
                    help="fused nested 4-bit dequant + linear vs dequant then cuBLAS, on the pull "
                         "request's public-path control shapes (one JSON line per case)")
    ap.add_argument("--nested-matrix", action="store_true",
                    help="fused vs three-launch nested dequant on the pull request's 24-cell matrix")
    ap.add_argument("--matrix", action="store_true",
                    help="the timed configuration cells besides c5: c1 (L2-resident), the c2 k-bit sweep "
                         "(K=2..5 x fp16/bf16/fp32) and the c4 nested blocksize sweep")
    ap.add_argument("--ref-seconds", type=float, default=120.0,
                    help="wall time the --impl reference run is sized for (all steps)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="target CPU time of the oracle baseline sample")
    return ap.parse_args()


# ----------------------------------------------------------------------------- workload

N_C5 = 16384 * 16384
NESTED_BS = 64


def op_bytes(kind, n, K=None, out_size=2, bs=NESTED_BS):
    """Algorithmic bytes of one launch (the minimum the operation must move)."""
    nb = (n + 31) // 32
    if kind == "quantize":
        return n * 2 + nb * K * 4 + nb * 4
    if kind == "dequantize":
        return nb * K * 4 + nb * 4 + n * out_size
    if kind == "quantize_e4m4":                   # one E4M4 byte of absmax per block
        return n * 2 + nb * K * 4 + nb
    if kind == "dequantize_e4m4":
        return nb * K * 4 + nb + n * out_size
    if kind in ("quantize_4bit", "quantize_nested"):
        bs = K or bs                              # these ops carry their outer blocksize as K
    nbo = (n + bs - 1) // bs
    nbi = (nbo + 255) // 256
    if kind == "quantize_4bit":                   # bf16 in; nibble codes and fp32 absmax out
        return n * 2 + (n + 1) // 2 + nbo * 4
    if kind == "quantize_nested":                 # bf16 in; codes, absmax_q, absmax2, offset out
        return n * 2 + (n + 1) // 2 + nbo + nbi * 4 + 4
    nbo = (n + bs - 1) // bs
    nbi = (nbo + 255) // 256
    return (n + 1) // 2 + nbo + nbi * 4 + n * out_size


ALL_OPS = [("quantize_k3", "quantize", 3), ("dequantize_k3", "dequantize", 3),
           ("quantize_k5", "quantize", 5), ("dequantize_k5", "dequantize", 5),
           ("nested_nf4_bs64", "nested", None)]
# Kernel launches per op (the nested quantize: 4-bit codes, two offset kernels, compression).
def nested_quant_launches(n, bs=NESTED_BS):
    """Launches of one quantize_4bit_nested call: the 4-bit codes, one per level of the offset
    tree while more than 2048 values remain, and the compression (which forms the root)."""
    count, levels = (n + bs - 1) // bs, 0
    while count > 2048:
        count = (count + 2047) // 2048
        levels += 1
    return 2 + levels

# Selectable with --ops (not part of the default step): the E4M4-absmax codec.
EXTRA_OPS = [(f"{k}_k{K}", k, K) for K in (2, 4) for k in ("quantize", "dequantize")] + \
    [(f"{k}_k{K}_e4m4", f"{k}_e4m4", K) for K in (3, 4, 5) for k in ("quantize", "dequantize")] + \
    [(f"quantize_4bit_nf4_bs{bs}", "quantize_4bit", bs) for bs in (64, 32)] + \
    [(f"quantize_nested_nf4_bs{bs}", "quantize_nested", bs) for bs in (64, 32)]


def workload_ops(only=None):
    if not only:
        return list(ALL_OPS)
    names = only.split(",")
    ops = [o for o in ALL_OPS + EXTRA_OPS if o[0] in names]
    assert len(ops) == len(names), f"unknown op in {only}"
    return ops


def workload_desc(n, ops, world=1):
    full = n == N_C5 and len(ops) == len(ALL_OPS)
    return {
        "parallelism": f"replicas{world}" if world > 1 else "single",
        "workload": ("c5: 16384x16384 bf16 weight ~ N(0,0.02) seed 7; k-bit quantize+dequantize at "
                     "K=3 and K=5 (blocksize 32, normal-float codebooks) and nested NF4 dequant "
                     "(outer blocksize 64, inner 256) of the same size, bf16 outputs")
        if full else f"c5-distributed subset: n={n}, ops={[o[0] for o in ops]} (profiling case)",
        "n": n, "io_dtype": "bf16", "blocksize": 32, "nested_blocksize": NESTED_BS,
        "l2": "no flush: every kernel streams >= 600 MB, above the 126 MB L2",
    }


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def _code_only(text):
    """Source text without comments and with whitespace collapsed: editing a comment leaves the
    hash of a kernel's source alone."""
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def kernel_source_hash(kind):
    files = {"quantize": ["kbit_quant.cu"], "dequantize": ["kbit_dequant.cu"],
             "quantize_e4m4": ["kbit_quant.cu"], "dequantize_e4m4": ["kbit_dequant.cu"],
             "quantize_4bit": ["kbit_quant.cu"], "quantize_nested": ["kbit_quant.cu", "nested_quant.cu"],
             "nested": ["nested_dequant.cu"]}[kind] + ["common.cuh"]
    h = hashlib.sha256()
    for f in files:
        h.update(_code_only(open(os.path.join(ROOT, "blockwise_bit_codebook_b200", "csrc", f)).read()).encode())
    return h.hexdigest()[:16]


def ncu_traffic(name, kind):
    """DRAM bytes per launch from the committed ncu summary, if the kernel source is unchanged."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p)).get(name)
    if not d or d.get("source_hash") != kernel_source_hash(kind):
        return None
    return d.get("dram_bytes_per_launch")


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.samples = []
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(gpu_index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), [s.strip() for s in line.split(",")]))

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0, t1):
        rows = [r for t, r in self.samples if t0 <= t <= t1 and len(r) >= 9]
        if not rows:
            rows = [r for t, r in self.samples if len(r) >= 9][-3:]
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": float(rows[0][2]) if rows[0][2].replace(".", "").isdigit() else None,
                "reasons": reasons, "samples": len(rows),
                "power_w_max": max([float(r[3]) for r in rows if r[3].replace(".", "").isdigit()],
                                   default=None)}


# ----------------------------------------------------------------------------- oracle legs

def oracle_sample_bytes_and_time(x_host_bits, cbs, nested, S):
    """Run the oracle over the first S elements of each input; returns (algorithmic bytes, seconds)."""
    import oracle
    codes, q, a2, off, code2, code4 = nested
    tot_bytes, t0 = 0, time.perf_counter()
    xs = x_host_bits[:S]
    for K in (3, 5):
        p, a = oracle.kbit_quantize(xs, "bf16", K, cbs[K])
        oracle.kbit_dequantize(p, a, cbs[K], K, S, "bf16")
        tot_bytes += op_bytes("quantize", S, K) + op_bytes("dequantize", S, K)
    nbo = (S + NESTED_BS - 1) // NESTED_BS
    oracle.nested_dequantize(codes[: (S + 1) // 2], q[:nbo], code2, a2[: (nbo + 255) // 256], off, code4,
                             S, NESTED_BS, 256, "bf16")
    tot_bytes += op_bytes("nested", S)
    return tot_bytes, time.perf_counter() - t0


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def oracle_parallel_time(x_host_bits, cbs, nested, S, threads):
    """The oracle over the first S elements of each input, split into `threads` contiguous ranges
    (multiples of 16384 elements: whole k-bit blocks and whole inner groups of the nested state)
    run at once, one thread each. The oracle's C functions are called through ctypes, which
    releases the interpreter lock, so the ranges run on separate cores. Returns (bytes, seconds)."""
    from concurrent.futures import ThreadPoolExecutor
    codes, q, a2, off, code2, code4 = nested
    unit = NESTED_BS * 256
    per = -(-S // threads // unit) * unit
    ranges = [(lo, min(S, lo + per)) for lo in range(0, S, per)]

    def one(r):
        lo, hi = r
        ns = (codes[lo // 2:], q[lo // NESTED_BS:], a2[lo // unit:], off, code2, code4)
        return oracle_sample_bytes_and_time(x_host_bits[lo:], cbs, ns, hi - lo)[0]

    with ThreadPoolExecutor(max_workers=len(ranges)) as ex:
        t0 = time.perf_counter()
        total = sum(ex.map(one, ranges))
        return total, time.perf_counter() - t0


def host_inputs_for_oracle(x_dev_bf16, nested_dev, code2, code4, S):
    import numpy as np
    import torch
    xb = x_dev_bf16[:S].contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    codes, q, a2, off = nested_dev
    nbo = (S + NESTED_BS - 1) // NESTED_BS
    return xb, (codes[: (S + 1) // 2].cpu().numpy(), q[:nbo].cpu().numpy(),
                a2[: (nbo + 255) // 256].cpu().numpy(), float(off), code2, code4)


def cpu_baseline(x_dev, nested_dev, code2, code4, cbs, seconds, n):
    # calibrate on 2^20 elements, then size the sample for about `seconds` of CPU work
    S0 = 1 << 20
    xb, ns = host_inputs_for_oracle(x_dev, nested_dev, code2, code4, S0)
    _, t = oracle_sample_bytes_and_time(xb, cbs, ns, S0)
    S = int(min(n, max(S0, S0 * seconds / max(t, 1e-3)))) // 4096 * 4096
    xb, ns = host_inputs_for_oracle(x_dev, nested_dev, code2, code4, S)
    b, t = oracle_sample_bytes_and_time(xb, cbs, ns, S)
    C = host_cores()
    bc, tc = oracle_parallel_time(xb, cbs, ns, S, C)
    return {"value": bc / tc / 1e9, "unit": "GB/s", "cores": C, "kind": "oracle",
            "seconds": round(tc, 2), "single_thread_value": b / t / 1e9, "single_thread_seconds": round(t, 2),
            "sample": f"first {S} of the {n} elements of every input (all five operations), the C oracle "
                      f"on {C} threads over contiguous ranges (and once on one thread)"}


# ----------------------------------------------------------------------------- main arm

def run_bbc(args):
    import numpy as np
    import torch

    import blockwise_bit_codebook_b200 as bbc
    from blockwise_bit_codebook_b200 import synthetic
    from blockwise_bit_codebook_b200.dist import max_over_ranks

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    bbc.load_library()

    ops = workload_ops(args.ops)
    n = args.n or N_C5
    nb = (n + 31) // 32
    x = synthetic.weights(n, std=0.02, seed=7, dtype=torch.bfloat16, device=dev)
    cbs = {K: bbc.bbc_nf_codebook(K) for K in (2, 3, 4, 5)}
    cb_dev = {K: torch.from_numpy(cbs[K]).to(dev) for K in cbs}
    ks = sorted({K for _, kind, K in ops if kind in ("quantize", "dequantize", "quantize_e4m4", "dequantize_e4m4")})
    nested = synthetic.nested_state(n, NESTED_BS, seed=3, device=dev)
    codes, q, a2, off = nested
    code2 = synthetic.general8_table()
    code4 = cbs[4]
    code2_dev, code4_dev = torch.from_numpy(code2).to(dev), cb_dev[4]
    kinds = {kind for _, kind, _ in ops}

    def make_outputs():
        """Every output (and workspace) buffer one step writes."""
        o = {"packed": {K: torch.empty(nb * K, dtype=torch.int32, device=dev) for K in ks},
             "absmax": {K: torch.empty(nb, dtype=torch.float32, device=dev) for K in ks},
             "absmax8": {K: torch.empty(nb, dtype=torch.uint8, device=dev) for K in ks},
             "outs": {K: torch.empty(n, dtype=torch.bfloat16, device=dev) for K in ks},
             "nout": torch.empty(n, dtype=torch.bfloat16, device=dev)}
        if kinds & {"quantize_4bit", "quantize_nested"}:
            bs4 = min(K for _, kind, K in ops if kind in ("quantize_4bit", "quantize_nested"))
            nbo4 = (n + bs4 - 1) // bs4
            o["q4_codes"] = torch.empty((n + 1) // 2, dtype=torch.uint8, device=dev)
            o["q4_absmax"] = torch.empty(nbo4, dtype=torch.float32, device=dev)
            o["nq_out"] = (torch.empty((n + 1) // 2, dtype=torch.uint8, device=dev),
                           torch.empty(nbo4, dtype=torch.uint8, device=dev),
                           torch.empty((nbo4 + 255) // 256, dtype=torch.float32, device=dev),
                           torch.empty(1, dtype=torch.float32, device=dev))
            o["nq_ws"] = torch.empty(bbc.quantize_4bit_nested_workspace_bytes(n, bs4), dtype=torch.uint8,
                                     device=dev)
        return o

    outA = make_outputs()
    inA = {"x": x, "codes": codes, "q": q, "a2": a2, "cb": cb_dev, "code4": code4_dev, "code2": code2_dev}
    stream = torch.cuda.current_stream(dev)

    def launch(kind, K, inp=inA, o=outA, st=stream):
        cb = inp["cb"]
        if kind == "quantize":
            bbc.kbit_quantize(inp["x"], K, cb[K], absmax=o["absmax"][K], packed=o["packed"][K], stream=st)
        elif kind == "dequantize":
            bbc.kbit_dequantize(o["packed"][K], o["absmax"][K], cb[K], K, n, torch.bfloat16, out=o["outs"][K],
                                stream=st)
        elif kind == "quantize_e4m4":
            bbc.kbit_quantize_e4m4(inp["x"], K, cb[K], absmax=o["absmax8"][K], packed=o["packed"][K], stream=st)
        elif kind == "dequantize_e4m4":
            bbc.kbit_dequantize_e4m4(o["packed"][K], o["absmax8"][K], cb[K], K, n, torch.bfloat16,
                                     out=o["outs"][K], stream=st)
        elif kind == "quantize_4bit":
            bbc.quantize_4bit(inp["x"], K, inp["code4"], absmax=o["q4_absmax"], codes=o["q4_codes"],
                              stream=st)
        elif kind == "quantize_nested":
            bbc.quantize_4bit_nested(inp["x"], K, inp["code4"], inp["code2"], workspace=o["nq_ws"],
                                     out=o["nq_out"], stream=st)
        else:
            bbc.dequantize_4bit_nested(inp["codes"], inp["q"], inp["code2"], inp["a2"], float(off), inp["code4"], n,
                                       NESTED_BS, torch.bfloat16, out=o["nout"], stream=st)

    for _ in range(args.warmup):
        for _, kind, K in ops:
            launch(kind, K)
    torch.cuda.synchronize()

    evs = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in ops]
           for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local) if rank == 0 else None
    time.sleep(0.3)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    w0 = time.time()
    t_start.record(stream)
    for s in range(args.steps):
        for i, (_, kind, K) in enumerate(ops):
            evs[s][i][0].record(stream)
            launch(kind, K)
            evs[s][i][1].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize()
    w1 = time.time()
    if dist:
        dist.barrier()
    total_ms = t_start.elapsed_time(t_end)
    samples = [[evs[s][i][0].elapsed_time(evs[s][i][1]) for s in range(args.steps)] for i in range(len(ops))]
    per_op_ms = [statistics.mean(v) for v in samples]

    def pct(v, q):
        v = sorted(v)
        return v[min(len(v) - 1, int(q * (len(v) - 1) + 0.5))]
    total_ms = max_over_ranks(total_ms, device=dev)      # identity at N = 1
    if sampler:
        time.sleep(0.25)
        sampler.stop()
    clocks = sampler.summary(w0, w1) if sampler else None

    ms_per_step = total_ms / args.steps
    bytes_step = sum(op_bytes(kind, n, K) for _, kind, K in ops)
    value = world * bytes_step / (ms_per_step * 1e-3) / 1e9
    peak, peak_kind = load_peaks()
    per_kernel = {}
    for (name, kind, K), ms, smp in zip(ops, per_op_ms, samples):
        b = op_bytes(kind, n, K)
        gbs = b / (ms * 1e-3) / 1e9
        per_kernel[name] = {"ms": round(ms, 5), "ms_p10_p50_p90": [round(pct(smp, q), 5) for q in (0.1, 0.5, 0.9)],
                            "GB/s": round(gbs, 1),
                            "Gelem/s": round(n / (ms * 1e-3) / 1e9, 2),
                            "frac_of_measured_hbm": round(gbs / peak, 4),
                            "frac_of_8TBs_nominal": round(gbs / 8000.0, 4),
                            "bytes_per_launch": b,
                            "share_of_step": round(ms / sum(per_op_ms), 4)}
    dom = max(range(len(ops)), key=lambda i: per_op_ms[i])
    dname, dkind, dK = ops[dom]
    dbytes = op_bytes(dkind, n, dK)
    achieved = dbytes / (per_op_ms[dom] * 1e-3) / 1e9
    roofline = {"bound": "hbm", "kernel": dname, "achieved": round(achieved, 1), "peak": peak,
                "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured"
                else "fallback 6.65 TB/s", "unit": "GB/s", "frac": round(achieved / peak, 4),
                "traffic": ncu_traffic(dname, dkind), "algorithmic_bytes_per_launch": dbytes}

    result = {"metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world,
              "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5),
              "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
              "data": "synthetic", "config": workload_desc(n, ops, world),
              "per_kernel": per_kernel, "roofline": roofline,
              "gpu_launches": sum(nested_quant_launches(n, K) if kind == "quantize_nested" else 1
                                  for _, kind, _ in ops) * args.steps, "clocks": clocks}

    # ---- end to end through the public API with host buffers
    if not args.no_e2e:
        # End to end through the public API from pinned host memory: every step copies its inputs
        # in and its results out inside the timed region. Two buffer sets and three streams (copies
        # in, compute, copies out, ordered by events) let step k + 1's input copies and kernels
        # overlap step k's output copies: PCIe carries the two directions at once.
        pin = lambda t: t.cpu().pin_memory()  # noqa: E731
        h_in = {"x": pin(x), "codes": pin(codes), "q": pin(q), "a2": pin(a2),
                "cb": {K: torch.from_numpy(cbs[K]).pin_memory() for K in (2, 3, 4, 5)}}
        k32 = sorted({K for _, kind, K in ops if kind in ("quantize", "dequantize")})
        k8 = sorted({K for _, kind, K in ops if kind.endswith("_e4m4")})

        def results(o):
            """The device tensors a step reads back (in a fixed order)."""
            r = [o["packed"][K] for K in ks] + [o["outs"][K] for K in ks] + [o["absmax"][K] for K in k32] + \
                [o["absmax8"][K] for K in k8] + [o["nout"]]
            if "quantize_4bit" in kinds:
                r += [o["q4_codes"], o["q4_absmax"]]
            if "quantize_nested" in kinds:
                r += list(o["nq_out"])
            return r

        sets = []
        for i in range(2):
            d_in = {"x": torch.empty_like(x), "codes": torch.empty_like(codes), "q": torch.empty_like(q),
                    "a2": torch.empty_like(a2), "cb": {K: torch.empty_like(cb_dev[K]) for K in (2, 3, 4, 5)}}
            d_in["code4"], d_in["code2"] = d_in["cb"][4], code2_dev
            sets.append((d_in, outA if i == 0 else make_outputs()))
        h_out = [torch.empty_like(t, device="cpu").pin_memory() for t in results(outA)]
        h2d = sum(h_in[k].numel() * h_in[k].element_size() for k in ("x", "codes", "q", "a2")) + \
            sum(t.numel() * 4 for t in h_in["cb"].values())
        d2h = sum(t.numel() * t.element_size() for t in h_out)
        s_in, s_comp, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_comp = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]

        def e2e_step(k):
            i = k % 2
            d_in, o = sets[i]
            s_in.wait_event(ev_comp[i])          # the set's inputs are no longer read
            with torch.cuda.stream(s_in):
                for key in ("x", "codes", "q", "a2"):
                    d_in[key].copy_(h_in[key], non_blocking=True)
                for K in (2, 3, 4, 5):
                    d_in["cb"][K].copy_(h_in["cb"][K], non_blocking=True)
                ev_in[i].record(s_in)
            s_comp.wait_event(ev_in[i])
            s_comp.wait_event(ev_out[i])         # the set's previous results have been read back
            for _, kind, K in ops:
                launch(kind, K, d_in, o, s_comp)
            ev_comp[i].record(s_comp)
            s_out.wait_event(ev_comp[i])
            with torch.cuda.stream(s_out):
                for h, t in zip(h_out, results(o)):
                    h.copy_(t, non_blocking=True)
                ev_out[i].record(s_out)

        for k in range(2):
            e2e_step(k)
        torch.cuda.synchronize()
        if dist:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s_in)
        for k in range(args.e2e_steps):
            e2e_step(k)
        e1.record(s_out)
        torch.cuda.synchronize()
        e_ms = max_over_ranks(e0.elapsed_time(e1) / args.e2e_steps, device=dev)
        result["e2e"] = {"value": round(world * bytes_step / (e_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
                         "ms_per_step": round(e_ms, 3), "h2d_bytes_per_step": h2d,
                         "d2h_bytes_per_step": d2h, "steps": args.e2e_steps,
                         "api": "blockwise_bit_codebook_b200 (C ABI via ctypes), pinned host buffers; copies in, "
                                "kernels and copies out on three streams, two buffer sets"}

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(x, nested, code2, code4, cbs, args.cpu_seconds, n)
    elif rank == 0:
        result["cpu_baseline"] = None

    if rank == 0 and world == 1 and not args.no_per_config and args.ops is None and n == N_C5:
        # the other configurations, each timed on its own after the c5 step (one GPU)
        torch.cuda.empty_cache()
        result["per_config"] = per_config_summary(config_cells(dev, peak))

    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


# ----------------------------------------------------------------------------- nested matrix

def run_linear(args):
    """Fused dequant + linear (linear_4bit_nested, linear_kbit) against the unfused sequence (the
    library's dequant into a materialised weight, then torch.matmul, i.e. cuBLAS) on the pull
    request's public-path control shapes: M = 1 and 8 (N = K = 4096) and M = 32 (N = 4096 and
    11008, K = 4096); bf16 activations; the nested NF4 weight (outer blocksize 64) and the k-bit
    K = 4 weight (blocksize 32). CUDA events around CUDA-graph replays of 200 repetitions (device
    time, no host launch overhead), alternating order, 7 rounds, medians. Two regimes: the same
    weight every call (it stays in L2, as in the page's timing loop) and "cold", where the calls
    cycle through copies of the weight state totalling more than L2. Algorithmic bytes of a fused
    call: the weight state, X and Y (the weight is never written)."""
    import torch

    import blockwise_bit_codebook_b200 as bbc
    from blockwise_bit_codebook_b200 import synthetic

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    bbc.load_library()
    peak, peak_kind = load_peaks()
    code4 = torch.from_numpy(bbc.bbc_nf_codebook(4)).to(dev)
    code2 = torch.from_numpy(synthetic.general8_table()).to(dev)
    bs = NESTED_BS
    KB = 4
    cbk = torch.from_numpy(bbc.bbc_nf_codebook(KB)).to(dev)
    shapes = [(1, 4096, 4096, "recurrent grad_A M=1"), (8, 4096, 4096, "recurrent grad_A M=8"),
              (32, 4096, 4096, "fallback forward M=32"), (32, 11008, 4096, "fallback forward M=32 N=11008"),
              (64, 4096, 4096, "batch M=64"), (128, 4096, 4096, "batch M=128"), (256, 4096, 4096, "batch M=256"),
              (256, 11008, 4096, "batch M=256 N=11008")]
    if args.linear_shapes:
        shapes = [s for s in shapes if s[0] in {int(m) for m in args.linear_shapes.split(",")}]
    for (M, N, K, label) in shapes:
        x = synthetic.weights(M * K, std=1.0, seed=4, dtype=torch.bfloat16, device=dev).reshape(M, K)
        w = torch.empty(N * K, dtype=torch.bfloat16, device=dev)
        y_f = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        y_u = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        for fmt in ("nested_nf4_bs64", f"kbit{KB}"):
            if fmt.startswith("nested"):
                codes, q, a2, off = synthetic.nested_state(N * K, bs, seed=3, device=dev)
                state = (codes, q)
                nbo = (N * K + bs - 1) // bs
                wbytes = N * K // 2 + nbo + ((nbo + 255) // 256) * 4

                def fused_on(c, qq):
                    bbc.linear_4bit_nested(x, c, qq, code2, a2, float(off), code4, N, bs, out=y_f)

                def unfused_on(c, qq):
                    bbc.dequantize_4bit_nested(c, qq, code2, a2, float(off), code4, N * K, bs, torch.bfloat16,
                                               out=w)
                    torch.matmul(x, w.view(N, K).t(), out=y_u)
            else:
                state = synthetic.kbit_state(N * K, KB, seed=3, device=dev)
                wbytes = N * K * KB // 8 + (N * K // 32) * 4

                def fused_on(pk, am):
                    bbc.linear_kbit(x, pk, am, cbk, KB, N, out=y_f)

                def unfused_on(pk, am):
                    bbc.kbit_dequantize(pk, am, cbk, KB, N * K, torch.bfloat16, out=w)
                    torch.matmul(x, w.view(N, K).t(), out=y_u)
            # "cold": the calls cycle through copies of the weight state that together exceed the
            # 126 MB L2, so every call reads its weight from HBM (as successive layers of a model do)
            ncopy = max(2, -(-160 * 2**20 // wbytes))
            copies = [tuple(t.clone() for t in state) for _ in range(ncopy)]
            for i in range(20):
                (fused_on if i % 2 == 0 else unfused_on)(*state)
            torch.cuda.synchronize()
            # Host-side call overhead (Python, ctypes) exceeds these kernels' device time, so each
            # variant's repetitions are captured once in a CUDA graph and the replays are timed.
            reps = 200
            graphs = {}
            for name, fn, cold in (("fused", fused_on, False), ("unfused", unfused_on, False),
                                   ("fused_cold", fused_on, True), ("unfused_cold", unfused_on, True)):
                gr = torch.cuda.CUDAGraph()
                with torch.cuda.graph(gr):
                    for r in range(reps):
                        fn(*(copies[r % ncopy] if cold else state))
                graphs[name] = gr
            torch.cuda.synchronize()
            samples = {k: [] for k in graphs}
            for rnd in range(7):
                order = list(graphs)
                if rnd % 2:
                    order.reverse()
                for name in order:
                    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    e0.record()
                    graphs[name].replay()
                    e1.record()
                    torch.cuda.synchronize()
                    samples[name].append(e0.elapsed_time(e1) / reps * 1e3)
            del graphs, copies
            med = {k: statistics.median(v) for k, v in samples.items()}
            nbytes = wbytes + M * K * 2 + M * N * 2
            rel = float((y_f.float() - y_u.float()).abs().max() / y_u.float().abs().max())
            flops = 2.0 * M * N * K
            print(json.dumps({"case": label, "format": fmt, "M": M, "N": N, "K": K, "dtype": "bf16",
                              "fused_TFLOPs": round(flops / med["fused"] / 1e6, 1),
                              "unfused_TFLOPs": round(flops / med["unfused"] / 1e6, 1),
                              "fused_us_median": round(med["fused"], 2), "unfused_us_median": round(med["unfused"], 2),
                              "unfused_over_fused": round(med["unfused"] / med["fused"], 3),
                              "fused_GBs": round(nbytes / med["fused"] / 1e3, 1),
                              "fused_frac_of_measured_hbm": round(nbytes / med["fused"] / 1e3 / peak, 4),
                              "cold_weight_copies": ncopy,
                              "fused_cold_us_median": round(med["fused_cold"], 2),
                              "unfused_cold_us_median": round(med["unfused_cold"], 2),
                              "cold_unfused_over_fused": round(med["unfused_cold"] / med["fused_cold"], 3),
                              "fused_cold_GBs": round(nbytes / med["fused_cold"] / 1e3, 1),
                              "fused_cold_frac_of_measured_hbm": round(nbytes / med["fused_cold"] / 1e3 / peak, 4),
                              "max_rel_diff_vs_unfused": round(rel, 6)}), flush=True)


def run_linear_case(args):
    """One fused-linear case for a profiler: the weight state of `--linear-case FMT:M[:N:K]` (FMT
    nested: NF4, outer blocksize 64, General8 absmax; kbit4: K = 4, blocksize 32, fp32 absmax),
    bf16 activations ~ N(0,1), then four calls of the public entry point."""
    import torch

    import blockwise_bit_codebook_b200 as bbc
    from blockwise_bit_codebook_b200 import synthetic

    parts = args.linear_case.split(":")
    fmt, M = parts[0], int(parts[1])
    N, K = (int(parts[2]), int(parts[3])) if len(parts) == 4 else (4096, 4096)
    dev = torch.device("cuda", 0)
    x = synthetic.weights(M * K, std=1.0, seed=4, dtype=torch.bfloat16, device=dev).reshape(M, K)
    if fmt == "nested":
        codes, q, a2, off = synthetic.nested_state(N * K, NESTED_BS, seed=3, device=dev)
        c4 = torch.from_numpy(bbc.bbc_nf_codebook(4)).to(dev)
        c2 = torch.from_numpy(synthetic.general8_table()).to(dev)

        def f():
            return bbc.linear_4bit_nested(x, codes, q, c2, a2, float(off), c4, N, NESTED_BS)
    elif fmt == "kbit4":
        pk, am = synthetic.kbit_state(N * K, 4, seed=3, device=dev)
        cb = torch.from_numpy(bbc.bbc_nf_codebook(4)).to(dev)

        def f():
            return bbc.linear_kbit(x, pk, am, cb, 4, N)
    else:
        raise SystemExit(f"unknown format {fmt} (nested or kbit4)")
    for _ in range(4):
        y = f()
    torch.cuda.synchronize()
    print(json.dumps({"linear_case": args.linear_case, "M": M, "N": N, "K": K,
                      "y_abs_sum": float(y.float().abs().sum())}), flush=True)


def _graph_time(fns, rounds=7):
    """Median, p10 and p90 device time (us) of one call, from CUDA-graph replays of `fns` (one
    call per element, cycling through buffer sets), 7 rounds."""
    import torch
    for f in fns[:4]:
        f()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for f in fns:
            f()
    torch.cuda.synchronize()
    samples = []
    for _ in range(rounds):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        g.replay()
        e1.record()
        torch.cuda.synchronize()
        samples.append(e0.elapsed_time(e1) / len(fns) * 1e3)
    del g
    return statistics.median(samples), pct_of(samples, 0.1), pct_of(samples, 0.9)


def _cell(cfg, op, dt_name, K, n, nbytes, t, nsets, peak, **extra):
    med, p10, p90 = t
    return {"config": cfg, "op": op, "dtype": dt_name, "K": K, "n": n, **extra,
            "us_median": round(med, 2), "us_p10_p90": [round(p10, 2), round(p90, 2)],
            "GB/s": round(nbytes / med / 1e3, 1), "Gelem/s": round(n / med / 1e3, 1),
            "frac_of_measured_hbm": round(nbytes / med / 1e3 / peak, 4), "buffer_sets": nsets}


def config_cells(dev, peak, c4_blocksizes=(64,), c4_formats=("nf4", "fp4"), c2_dtypes=None):
    """The timed configuration cells other than the c5 step, as a list of dicts.

    c1: 1,048,576 fp32 ~ N(0,1) (seed 0), K=4 quantize and dequantize to fp32: 4.9 MB, so
        L2-resident: reported as latency, not against the HBM roofline.
    c2: 4096x4096 ~ N(0,0.02) (seed 1) with 0.1 % outliers x20 (seed 2), K = 2..5 x fp16 / bf16 /
        fp32, quantize then dequantize; every cell cycles through >= 4 buffer sets holding more
        than twice the 126 MB L2, so each launch streams from HBM.
    c3: nested NF4 dequant of 4096x11008 (outer blocksize 64), fp16 / bf16 / fp32 outputs.
    c4: nested dequant of 8192x8192 (every General8 code present, all 16 value codes) at the
        given outer blocksizes and formats, bf16 and fp32 outputs (>= 168 MB per launch).
    Each cell: CUDA-graph replays of back-to-back calls (one per buffer set; host launch cost
    excluded), 7 rounds, median / p10 / p90; GB/s = algorithmic bytes / median time."""
    import torch

    import blockwise_bit_codebook_b200 as bbc
    from blockwise_bit_codebook_b200 import synthetic

    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    sizes = {torch.float16: 2, torch.bfloat16: 2, torch.float32: 4}
    names = {torch.float16: "fp16", torch.bfloat16: "bf16", torch.float32: "fp32"}
    cells = []

    def kbit_cells(cfg, n, dt, Ks, x0, l2_resident, reps_per_set):
        s_in = sizes[dt]
        nb = (n + 31) // 32
        for K in Ks:
            cb = torch.from_numpy(bbc.bbc_nf_codebook(K)).to(dev)
            qb = n * s_in + nb * K * 4 + nb * 4
            nsets = 1 if l2_resident else max(4, -(-2 * l2 // qb))
            xs = [x0.clone() for _ in range(nsets)]
            packed = [torch.empty(nb * K, dtype=torch.int32, device=dev) for _ in range(nsets)]
            absmax = [torch.empty(nb, dtype=torch.float32, device=dev) for _ in range(nsets)]
            outs = [torch.empty(n, dtype=dt, device=dev) for _ in range(nsets)]
            qf = [(lambda i=i: bbc.kbit_quantize(xs[i], K, cb, absmax=absmax[i], packed=packed[i]))
                  for i in range(nsets)] * reps_per_set
            cells.append(_cell(cfg, "quantize", names[dt], K, n, qb, _graph_time(qf), nsets, peak))
            df = [(lambda i=i: bbc.kbit_dequantize(packed[i], absmax[i], cb, K, n, dt, out=outs[i]))
                  for i in range(nsets)] * reps_per_set
            cells.append(_cell(cfg, "dequantize", names[dt], K, n, qb, _graph_time(df), nsets, peak))
            del xs, packed, absmax, outs
            torch.cuda.empty_cache()

    def nested_cells(cfg, n, bs, fmts, dts, seed, all_codes, reps):
        codes, q, a2, off = synthetic.nested_state(n, bs, seed=seed, device=dev, all_codes=all_codes)
        code2 = torch.from_numpy(synthetic.general8_table()).to(dev)
        tabs = {"nf4": bbc.bbc_nf_codebook(4), "fp4": synthetic.fp4_table()}
        for fmt in fmts:
            code4 = torch.from_numpy(tabs[fmt]).to(dev)
            for dt in dts:
                # inputs and outputs both rotate through sets holding more than twice the L2
                nbytes = op_bytes("nested", n, out_size=sizes[dt], bs=bs)
                nsets = max(2, -(-2 * l2 // nbytes))
                sets = [(codes.clone(), q.clone(), a2.clone(), torch.empty(n, dtype=dt, device=dev))
                        for _ in range(nsets)]
                fns = [(lambda s=s: bbc.dequantize_4bit_nested(s[0], s[1], code2, s[2], float(off), code4, n, bs, dt,
                                                               out=s[3])) for s in sets] * reps
                cells.append(_cell(cfg, "nested_dequant", names[dt], None, n, nbytes, _graph_time(fns), nsets, peak,
                                   format=fmt, blocksize=bs))
                del sets
        del codes, q, a2
        torch.cuda.empty_cache()

    # c1: L2-resident, one buffer set
    n1 = 1 << 20
    x1 = synthetic.weights(n1, std=1.0, seed=0, dtype=torch.float32, device=dev)
    kbit_cells("c1", n1, torch.float32, [4], x1, True, 200)
    # c2: the k-bit sweep
    n2 = 4096 * 4096
    for dt in (c2_dtypes or (torch.float16, torch.bfloat16, torch.float32)):
        x2 = synthetic.weights(n2, std=0.02, seed=1, dtype=dt, device=dev, outlier_frac=0.001)
        kbit_cells("c2", n2, dt, [2, 3, 4, 5], x2, False, 8)
        del x2
    # c3: the headline nested cell (the output buffers rotate so writes do not stay in L2)
    nested_cells("c3", 4096 * 11008, 64, ("nf4",), (torch.float16, torch.bfloat16, torch.float32), 3, False, 10)
    # c4: 8192x8192 at the given outer blocksizes
    for bs in c4_blocksizes:
        nested_cells("c4", 8192 * 8192, bs, c4_formats, (torch.bfloat16, torch.float32), 3, True, 10)
    return cells


def run_matrix(args):
    """Every timed configuration cell besides the c5 step (config_cells), the c4 sweep over all
    six outer blocksizes, one JSON line per cell."""
    import torch

    import blockwise_bit_codebook_b200 as bbc

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    bbc.load_library()
    peak, _ = load_peaks()
    for c in config_cells(dev, peak, c4_blocksizes=(32, 64, 128, 256, 1024, 4096)):
        print(json.dumps(c), flush=True)


def per_config_summary(cells):
    """The default line's per_config block: every cell by name, and the lowest fraction of the
    measured HBM copy bandwidth per (config, op) over the HBM-bound configurations."""
    out, lows = {}, {}
    for c in cells:
        name = ":".join(str(x) for x in (c["config"], c["op"], c["dtype"], f"K{c['K']}" if c["K"] else None,
                                         c.get("format"), f"bs{c['blocksize']}" if c.get("blocksize") else None)
                        if x)
        out[name] = {"us": c["us_median"], "GB/s": c["GB/s"], "Gelem/s": c["Gelem/s"],
                     "frac_of_measured_hbm": c["frac_of_measured_hbm"], "buffer_sets": c["buffer_sets"]}
        if c["config"] != "c1":
            key = f"{c['config']}:{c['op']}"
            lows[key] = min(lows.get(key, 1e9), c["frac_of_measured_hbm"])
    return {"cells": out, "min_frac_of_measured_hbm": lows,
            "method": "CUDA-graph replays of back-to-back calls over rotating buffer sets (> 2x L2 for c2, "
                      "c3, c4), 7 rounds, medians; c1 is L2-resident (latency, not an HBM fraction)"}


def run_nested_matrix(args):
    """Fused nested dequant vs the unfused three-launch chain on the pull request's matrix.

    Shapes 4096x4096, 11008x4096, 4096x11008, 8192x8192; NF4 and FP4; fp16/bf16/fp32 outputs;
    outer blocksize 64. Method as the pull request describes it: CUDA events, 20 alternating
    warm-ups, 7 interleaved rounds of size-scaled repetitions (up to 100), medians; outputs are
    checked bit-equal. Inputs are not flushed from L2 between repetitions (as there).
    """
    import math

    import numpy as np
    import torch

    import blockwise_bit_codebook_b200 as bbc
    from blockwise_bit_codebook_b200 import synthetic

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    bbc.load_library()
    shapes = [(4096, 4096), (11008, 4096), (4096, 11008), (8192, 8192)]
    tabs = {"nf4": bbc.bbc_nf_codebook(4), "fp4": synthetic.fp4_table()}
    code2 = torch.from_numpy(synthetic.general8_table()).to(dev)
    bs = 64
    ratios = {}
    for (r, c) in shapes:
        n = r * c
        codes, q, a2, off = synthetic.nested_state(n, bs, seed=3, device=dev)
        ws = torch.empty((n + bs - 1) // bs, dtype=torch.float32, device=dev)
        for fmt in ("nf4", "fp4"):
            code4 = torch.from_numpy(tabs[fmt]).to(dev)
            for dt in (torch.float16, torch.bfloat16, torch.float32):
                out_f = torch.empty(n, dtype=dt, device=dev)
                out_c = torch.empty(n, dtype=dt, device=dev)
                fused = lambda: bbc.dequantize_4bit_nested(codes, q, code2, a2, float(off), code4, n, bs, dt,  # noqa: E731
                                                           out=out_f)
                chain = lambda: bbc.dequantize_4bit_nested_chain(codes, q, code2, a2, float(off), code4, n,  # noqa: E731
                                                                 bs, dt, out=out_c, scale_workspace=ws)
                for i in range(20):
                    (fused if i % 2 == 0 else chain)()
                torch.cuda.synchronize()
                nbytes = op_bytes("nested", n, out_size=out_f.element_size())
                reps = max(10, min(100, int(4e9 / nbytes)))
                samples = {"fused": [], "chain": []}
                for rnd in range(7):
                    order = [("fused", fused), ("chain", chain)]
                    if rnd % 2:
                        order.reverse()
                    for name, fn in order:
                        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                        e0.record()
                        for _ in range(reps):
                            fn()
                        e1.record()
                        torch.cuda.synchronize()
                        samples[name].append(e0.elapsed_time(e1) / reps * 1e3)
                equal = bool(torch.equal(out_f.view(torch.int16 if dt != torch.float32 else torch.int32),
                                         out_c.view(torch.int16 if dt != torch.float32 else torch.int32)))
                med = {k: statistics.median(v) for k, v in samples.items()}
                ratio = med["chain"] / med["fused"]
                ratios.setdefault(f"{r}x{c}", []).append(ratio)
                print(json.dumps({"cell": f"{r}x{c}", "format": fmt, "dtype": str(dt).split(".")[-1],
                                  "blocksize": bs, "fused_us_median": round(med["fused"], 2),
                                  "chain_us_median": round(med["chain"], 2),
                                  "fused_us_p10_p90": [round(pct_of(samples["fused"], 0.1), 2),
                                                       round(pct_of(samples["fused"], 0.9), 2)],
                                  "chain_us_p10_p90": [round(pct_of(samples["chain"], 0.1), 2),
                                                       round(pct_of(samples["chain"], 0.9), 2)],
                                  "fused_GBs": round(nbytes / med["fused"] / 1e3, 1),
                                  "chain_over_fused": round(ratio, 4), "bit_equal": equal}), flush=True)
    geo = lambda v: math.exp(sum(math.log(x) for x in v) / len(v))  # noqa: E731
    allr = [x for v in ratios.values() for x in v]
    print(json.dumps({"summary": "chain/fused geomean per shape (outer blocksize 64)",
                      "per_shape": {k: round(geo(v), 4) for k, v in ratios.items()},
                      "all_cells": round(geo(allr), 4), "min": round(min(allr), 4),
                      "max": round(max(allr), 4), "cells": len(allr)}), flush=True)


def pct_of(v, q):
    v = sorted(v)
    return v[min(len(v) - 1, int(q * (len(v) - 1) + 0.5))]


# ----------------------------------------------------------------------------- reference arm

def run_reference(args):
    """The CPU oracle as the reference arm: rank 0 only, bounded samples of the c5 workload."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import numpy as np
    import torch

    import oracle
    from blockwise_bit_codebook_b200 import synthetic

    n = N_C5
    cbs = {K: oracle.normal_float_codebook(K) for K in (3, 4, 5)}
    code2 = synthetic.general8_table()
    # per-step sample sized so the whole run takes about two minutes, all host cores busy
    C = host_cores()
    budget = args.ref_seconds / max(1, args.steps + args.warmup)
    S = max(16384, min(n, int(budget * C / 170e-9)) // 16384 * 16384)
    x = synthetic.weights(S, std=0.02, seed=7, dtype=torch.bfloat16)
    xb = x.view(torch.int16).numpy().view(np.uint16)
    codes, q, a2, off = synthetic.nested_state(S, NESTED_BS, seed=3)
    ns = (codes.numpy(), q.numpy(), a2.numpy(), float(off), code2, cbs[4])
    for _ in range(args.warmup):
        oracle_parallel_time(xb, cbs, ns, S, C)
    tot_b, tot_t = 0, 0.0
    for _ in range(args.steps):
        b, t = oracle_parallel_time(xb, cbs, ns, S, C)
        tot_b += b
        tot_t += t
    value = tot_b / tot_t / 1e9
    sample = (f"{S} elements per step (first elements of a c5-distributed input), all five operations, "
              f"the C oracle on {C} threads over contiguous ranges")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(tot_t / args.steps * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": workload_desc(N_C5, ALL_OPS, int(os.environ.get("WORLD_SIZE", "1"))),
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": C, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def relaunch_under_torchrun(args):
    """`bench.py --gpus N` (N > 1) started without torchrun starts N ranks itself, one per GPU, as
    the driver does (torchrun on 127.0.0.1); rank 0 prints the line."""
    import subprocess
    import sys
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={args.gpus}",
           "--master-addr", "127.0.0.1", "--master-port", os.environ.get("BBC_BENCH_PORT", "29513"),
           os.path.abspath(__file__), *sys.argv[1:]]
    sys.exit(subprocess.call(cmd))


if __name__ == "__main__":
    a = parse_args()
    if a.gpus > 1 and "WORLD_SIZE" not in os.environ and a.impl == "bbc" and not (
            a.linear or a.linear_case or a.matrix or a.nested_matrix):
        relaunch_under_torchrun(a)
    world_env = int(os.environ.get("WORLD_SIZE", "1"))
    if a.impl == "bbc" and "WORLD_SIZE" in os.environ and world_env != a.gpus:
        raise SystemExit(f"--gpus {a.gpus} but WORLD_SIZE={world_env}: start one rank per GPU")
    if a.linear_case:
        run_linear_case(a)
    elif a.linear:
        run_linear(a)
    elif a.matrix:
        run_matrix(a)
    elif a.nested_matrix:
        run_nested_matrix(a)
    elif a.impl == "reference":
        run_reference(a)
    else:
        run_bbc(a)
