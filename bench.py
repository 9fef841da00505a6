#!/usr/bin/env python
"""GPTQ layer-quantization throughput on B200.

One step = the whole per-layer pass on one synthetic layer resident in HBM:
  H = 2/N X^T X (tcgen05 SYRK) -> damping + U (Cholesky, triangular inverse)
  -> the GPTQ column loop (lazy 128-column blocks + trailing updates)
  -> packing of codes and zero points.
Default workload: a Llama-7B attention projection, W 4096x4096 bf16 and X
262,144 tokens x 4096 bf16 (the X stream alone is 2.15 GB, larger than L2),
4-bit, group 128, damp 0.01, block 128.

N GPUs (torchrun): every rank quantizes its own layer (a different seed); no
collective on the data path (weak scaling); time = max over ranks.

--workload layerset_block: one step = one block of the 7B-shaped layer set
(q, k, v, o 4096x4096; gate, up 11008x4096; down 4096x11008; one X of 131,072
tokens per input group, H and U shared by q/k/v and by gate/up), 4-bit g128;
the 32-block set takes 32 times a block.

--impl reference times the fp64 CPU oracle (the only reference: the method's
pages publish no code) on a bounded sample of the same workload.
"""
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

METRIC = "GPTQ layer quant: weights/sec and ms per 4096×4096 layer; % of roofline"
UNIT = "weights/s"
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="attn4096")
    ap.add_argument("--tokens", type=int, default=None,
                    help="override the calibration token count (small profiling captures only)")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-gptq2d", action="store_true", help="skip the GPTQ-2D measurement")
    ap.add_argument("--no-others", action="store_true", help="skip the other synthetic workloads")
    ap.add_argument("--profile-pass", action="store_true",
                    help="no timing: two small layer passes (4096x4096, 32,768 tokens) and 8 packed matvecs, "
                         "for kernel-by-kernel ncu captures")
    ap.add_argument("--cpu-tokens", type=int, default=4096, help="oracle sample: tokens for H")
    ap.add_argument("--cpu-rows", type=int, default=32, help="oracle sample: rows through the column loop")
    return ap.parse_args()


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def rank_seed(seed, rank):
    """Each rank quantizes its own layer: a distinct seed per rank."""
    return seed + 7919 * rank


def max_over_ranks(value, dist, device):
    """The slowest rank's time (every rank receives it); `dist` is None for one
    process."""
    if dist is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(world, rows, n, ms):
    """Whole-job weights per second: every rank's layer over the slowest time."""
    return world * rows * n / (ms / 1e3)


def stage_rooflines(stage_ms, rows, n, bits, ng, pk):
    """Roofline fractions of the non-SYRK stages from their CUDA-event times.

    factorization (damping, act-order, Cholesky and triangular inverse on the
    tensor cores, the anti-transpose): 2 n^3 / 3 fp32-accurate flops against
    the bf16 tensor peak, and the tf32 issue rate (3 MMAs per product) against
    the tf32 peak; packing: the codes and zero points read (1 byte each) and
    their packed words written, against the HBM copy rate.
    """
    t_factor = stage_ms["prepare_hinv"] / 1e3
    t_pack = stage_ms["pack"] / 1e3
    tf32_peak = pk["bf16_tflops"] * 1.1 / 2.25
    factor_tflops = 2.0 * n ** 3 / 3.0 / t_factor / 1e12
    words = lambda k: bits * ((k + 31) // 32)
    pack_bytes = rows * n + rows * ng + 4 * rows * (words(n) + words(ng))
    pack_gbs = pack_bytes / t_pack / 1e9
    return {"factorization": {"bound": "tensor", "achieved": factor_tflops, "peak": pk["bf16_tflops"],
                              "unit": "TFLOP/s", "frac": factor_tflops / pk["bf16_tflops"],
                              "tf32_issue_frac": 3 * factor_tflops / tf32_peak,
                              "peak_source": "measured bf16 burst; tf32 = that x 1.1 / 2.25 (nominal ratio)"},
            "pack": {"bound": "hbm", "achieved": pack_gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                     "frac": pack_gbs / pk["hbm_gbs"], "algorithmic_bytes": pack_bytes}}


def trailing_flops(rows, n, block):
    """Algorithmic flops of the lazy trailing updates: every block's errors
    times the rows of U right of it, 2 rows (i2 - i1) (n - i2) per block
    (the two-level schedule does the same products in another order)."""
    total = 0
    for i1 in range(0, n, block):
        i2 = min(i1 + block, n)
        total += 2 * rows * (i2 - i1) * (n - i2)
    return float(total)


def kernel_rooflines(trace, steps, rows, n, n_tok, bits, ng, block, pk, sms, mhz):
    """Per-kernel achieved rates from a traced pass (CUDA events around each
    launch, gptq_trace_read), each against its roofline."""
    def ms(name):
        hits = [v for k, v in trace.items() if k == name or k.startswith(name + "<")]
        return sum(v[1] for v in hits) / steps, sum(v[0] for v in hits) / steps

    tf32_peak = pk["bf16_tflops"] * 1.1 / 2.25  # tf32 from the measured bf16 peak by the nominal ratio
    fma_peak = sms * 128 * 2 * mhz * 1e6 / 1e12
    out = {}
    t, l = ms("syrk_tc_kernel")
    if t > 0:
        f = float(n) * (n + 1) * n_tok
        out["syrk_tc_kernel"] = {"bound": "tensor", "ms": t, "launches": l, "achieved": f / t / 1e9,
                                 "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                                 "frac": f / t / 1e9 / pk["bf16_tflops"], "algorithmic_flops": f}
    t, l = ms("chol_tc_kernel")
    if t > 0:
        f = 2.0 * n ** 3 / 3.0
        a = f / t / 1e9
        out["chol_tc_kernel"] = {"bound": "tensor", "ms": t, "launches": l, "achieved": a, "unit": "TFLOP/s",
                                 "peak": pk["bf16_tflops"], "frac": a / pk["bf16_tflops"],
                                 "tf32_issue_frac": 3 * a / tf32_peak, "algorithmic_flops": f,
                                 "note": "2n^3/3 fp32-accurate flops (Cholesky + triangular inverse); each product "
                                         "is 3 tf32 MMAs, so tf32_issue_frac = 3 x achieved / tf32 peak"}
    t, l = ms("trailing_tc_kernel")
    if t > 0:
        f = trailing_flops(rows, n, block)
        a = f / t / 1e9
        out["trailing_tc_kernel"] = {"bound": "tensor", "ms": t, "launches": l, "achieved": a, "unit": "TFLOP/s",
                                     "peak": pk["bf16_tflops"], "frac": a / pk["bf16_tflops"],
                                     "tf32_issue_frac": 3 * a / tf32_peak, "algorithmic_flops": f,
                                     "note": "fp32-accurate products, 3 tf32 MMAs each"}
    t, l = ms("gptq_block_kernel")
    if t > 0:
        # reads the working weights and U's diagonal tiles; writes the errors
        # (tf32 hi and lo), the codes and the group parameters
        b = rows * n * 4 + n * block * 4 + rows * n * 8 + rows * n + rows * ng * 5
        out["gptq_block_kernel"] = {"bound": "latency", "ms": t, "launches": l, "achieved": b / t / 1e6,
                                    "unit": "GB/s", "peak": pk["hbm_gbs"], "frac": b / t / 1e6 / pk["hbm_gbs"],
                                    "algorithmic_bytes": b,
                                    "note": "a 128-step dependent chain per row and block; HBM fraction for context"}
    t, l = ms("pack_kernel")
    if t > 0:
        words = lambda k: bits * ((k + 31) // 32)
        b = rows * n + rows * ng + 4 * rows * (words(n) + words(ng))
        out["pack_kernel"] = {"bound": "hbm", "ms": t, "launches": l, "achieved": b / t / 1e6, "unit": "GB/s",
                              "peak": pk["hbm_gbs"], "frac": b / t / 1e6 / pk["hbm_gbs"], "algorithmic_bytes": b}
    for name in ("syrk_finalize_kernel", "gather_reversed_kernel", "anti_transpose_kernel", "gather_weights_kernel",
                 "split_transpose_tf32_kernel", "outputs_kernel", "diag_prep_kernel"):
        t, l = ms(name)
        if t > 0:
            out[name] = {"ms": t, "launches": l}
    return out


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK}, "measured"
    except Exception:
        return dict(FALLBACK), "fallback"


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    """nvidia-smi samples (every 100 ms) of the GPU a process runs on."""

    QUERY = ("index,uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid):
        self.uuid = (uuid or "").lower()
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                                          "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        rows = []
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 10:
                continue
            if self.uuid and self.uuid not in f[1].lower():
                continue
            try:
                rows.append({"sm": float(f[2]), "max": float(f[3]), "power": float(f[4]),
                             "hw_slowdown": f[6], "hw_thermal": f[7], "sw_thermal": f[8], "sw_power_cap": f[9]})
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        loaded = [r for r in rows if r["power"] > 300.0] or rows
        reasons = set()
        names = {"hw_thermal": "hw_thermal_slowdown", "sw_thermal": "sw_thermal_slowdown"}
        for r in loaded:
            for k in ("hw_slowdown", "hw_thermal", "sw_thermal", "sw_power_cap"):
                if r[k].lower() == "active":
                    reasons.add(names.get(k, k))
        return {"sm_mhz": statistics.median(r["sm"] for r in loaded), "sm_max_mhz": max(r["max"] for r in rows),
                "reasons": sorted(reasons), "samples": len(loaded)}


# ---------------------------------------------------------------------------
# CPU oracle on a bounded sample
# ---------------------------------------------------------------------------

def oracle_sample(W_host, X_host, spec, tokens, rows):
    """Times the fp64 oracle on a sample and scales each stage to the full layer.

    H: `tokens` of the N tokens (cost grows with tokens) -> x N/tokens.
    U: the full n x n factor (computed in full).
    Column loop + packing: `rows` of the rows (rows are independent) -> x rows_total/rows.
    """
    import numpy as np

    from oracle import gptq_oracle as go

    n = spec.n
    Xs = X_host[:tokens].double().numpy()
    Ws = W_host[:rows].double().numpy()
    t0 = time.perf_counter()
    H = go.hessian(Xs, alpha=2.0 / tokens)
    t1 = time.perf_counter()
    prep = go.prepare(H, Ws, spec.damp, spec.act_order)
    U = go.inverse_factor(prep["H"])
    t2 = time.perf_counter()
    res = go.gptq_quantize(prep["W"], U, spec.bits, spec.group, spec.block)
    go.pack_codes(res["codes"], spec.bits)
    t3 = time.perf_counter()
    s_h = spec.n_tok / tokens
    s_q = spec.rows / rows
    full = (t1 - t0) * s_h + (t2 - t1) + (t3 - t2) * s_q
    threads = None
    try:
        from threadpoolctl import threadpool_info
        threads = max((i.get("num_threads") or 0) for i in threadpool_info()) or None
    except Exception:
        pass
    cores = threads or len(os.sched_getaffinity(0))
    sample = (f"fp64 oracle on {tokens} of {spec.n_tok} tokens for H (time x{s_h:g}), the full {n}x{n} factor, "
              f"{rows} of {spec.rows} rows through the column loop and packing (time x{s_q:g}); "
              f"measured {t3 - t0:.2f} s")
    return {"value": spec.rows * n / full, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample,
            "est_s_per_layer": full, "stage_s": {"hessian_sample": t1 - t0, "factor": t2 - t1,
                                                  "loop_and_pack_sample": t3 - t2}}


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def kernel_source_hash():
    h = hashlib.sha256()
    with open(os.path.join(ROOT, "post_weight_quantization_accum_b200", "csrc", "hessian.cu"), "rb") as f:
        h.update(f.read())
    return h.hexdigest()[:16]


def measured_traffic(workload):
    """Per-launch DRAM bytes of the SYRK kernel from an ncu capture, if it is
    still the kernel that was captured (else None)."""
    path = os.path.join(ROOT, "profiles", f"syrk_tc_kernel.{workload}.traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        if d.get("hessian_cu_sha256_16") == kernel_source_hash():
            return float(d["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


class LayerPass:
    """One layer pass (H, U, column loop, packing) through the library calls on
    preallocated buffers, with CUDA events between the stages."""

    nev = 5

    def __init__(self, gq, spec, W, X, dev):
        import torch

        self.gq, self.spec, self.W, self.X, self.dev = gq, spec, W, X, dev
        n, rows = spec.n, spec.rows
        ng = gq.LIB.gptq_num_groups(n, spec.group)
        self.alpha = 2.0 / spec.n_tok
        self.H = torch.zeros((n, n), dtype=torch.float32, device=dev)
        self.hdiag = torch.zeros(n, dtype=torch.float64, device=dev) if spec.act_order else None
        self.U = torch.empty((n, n), dtype=torch.float32, device=dev)
        self.perm = torch.empty(n, dtype=torch.int32, device=dev)
        self.dead = torch.empty(n, dtype=torch.uint8, device=dev)
        self.out = {"codes": torch.empty((rows, n), dtype=torch.uint8, device=dev),
                    "scales": torch.empty((rows, ng), dtype=torch.float32, device=dev),
                    "zeros": torch.empty((rows, ng), dtype=torch.uint8, device=dev),
                    "g_idx": torch.empty(n, dtype=torch.int32, device=dev)}
        self.packed = torch.empty((rows, gq.LIB.gptq_packed_words_per_row(n, spec.bits)), dtype=torch.int32,
                                  device=dev)
        self.packed_z = torch.empty((rows, gq.LIB.gptq_packed_words_per_row(ng, spec.bits)), dtype=torch.int32,
                                    device=dev)
        self.ws_h = gq.workspace(gq.LIB.gptq_hessian_workspace_size(n, spec.n_tok), dev)
        self.ws_p = gq.workspace(gq.LIB.gptq_prepare_workspace_size(n), dev)
        self.ws_q = gq.workspace(gq.LIB.gptq_quantize_workspace_size(rows, n, spec.block), dev)
        self.stream = torch.cuda.current_stream()

    def new_events(self):
        import torch

        return [torch.cuda.Event(enable_timing=True) for _ in range(self.nev)]

    def step(self, evs):
        gq, spec, st = self.gq, self.spec, self.stream
        self.H.zero_()
        if self.hdiag is not None:
            self.hdiag.zero_()
        evs[0].record(st)
        gq.gptq_hessian_accum(self.H, self.X, self.alpha, hdiag=self.hdiag, ws=self.ws_h)
        evs[1].record(st)
        gq.gptq_prepare_hinv(self.H, spec.damp, spec.act_order, hdiag=self.hdiag, perm=self.perm, dead=self.dead,
                             U=self.U, ws=self.ws_p)
        evs[2].record(st)
        gq.gptq_quantize_layer(self.W, self.U, spec.bits, spec.group, spec.block,
                               perm=self.perm if spec.act_order else None, dead=self.dead, out=self.out, ws=self.ws_q)
        evs[3].record(st)
        gq.gptq_pack(self.out["codes"], spec.bits, packed=self.packed)
        gq.gptq_pack(self.out["zeros"], spec.bits, packed=self.packed_z)
        evs[4].record(st)


def measure_workload(gq, si, name, dev, steps=2, warmup=1, pk=None, sms=148, mhz=1965.0):
    """A few timed layer passes of another synthetic layer (its own inputs,
    freed afterwards): per-layer time, weights/s, stage times and per-kernel
    rooflines from one traced pass."""
    import torch

    spec = si.SPECS[name]
    W, X = si.make_layer(spec, dev)
    lp = LayerPass(gq, spec, W, X, dev)
    for _ in range(warmup):
        lp.step(lp.new_events())
    torch.cuda.synchronize()
    evs = [lp.new_events() for _ in range(steps)]
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(lp.stream)
    for k in range(steps):
        lp.step(evs[k])
    e.record(lp.stream)
    torch.cuda.synchronize()
    ms = s.elapsed_time(e) / steps
    stage = [statistics.mean(ev[i].elapsed_time(ev[i + 1]) for ev in evs) for i in range(lp.nev - 1)]
    gq.gptq_trace_read()
    gq.gptq_trace_enable(True)
    lp.step(lp.new_events())
    torch.cuda.synchronize()
    trace = gq.gptq_trace_read()
    gq.gptq_trace_enable(False)
    status = gq.gptq_get_device_status()
    ng = gq.LIB.gptq_num_groups(spec.n, spec.group)
    res = {"workload": f"W {spec.rows}x{spec.n} {spec.w_dtype}, X {spec.n_tok} tokens ({spec.x_kind}), "
                       f"{spec.bits}-bit group {spec.group}, act_order {spec.act_order}",
           "ms_per_layer": ms, "weights_per_s": spec.rows * spec.n / (ms / 1e3), "steps": steps,
           "stages_ms": dict(zip(("hessian", "prepare_hinv", "quantize_layer", "pack"), stage)),
           "kernel_rooflines": kernel_rooflines(trace, 1, spec.rows, spec.n, spec.n_tok, spec.bits, ng, spec.block,
                                                pk, sms, mhz),
           "device_status": status}
    del lp, W, X
    torch.cuda.empty_cache()
    return res


def run_ours(args, world, rank, local):
    import torch

    import post_weight_quantization_accum_b200 as gq
    import synth_inputs as si

    dist = None
    if world > 1:
        import torch.distributed as dist
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())
    base = si.SPECS[args.workload]
    spec = si.scaled(base, seed=rank_seed(base.seed, rank), n_tok=args.tokens or base.n_tok)
    W, X = si.make_layer(spec, dev)
    n, rows = spec.n, spec.rows
    ng = gq.LIB.gptq_num_groups(n, spec.group)
    lp = LayerPass(gq, spec, W, X, dev)
    stream = lp.stream
    step, new_events, nev = lp.step, lp.new_events, lp.nev
    out, packed = lp.out, lp.packed

    for _ in range(args.warmup):
        step(new_events())
    torch.cuda.synchronize()
    st = gq.gptq_get_device_status()
    if st != 0:
        raise RuntimeError(f"device status after warm-up: {st}")

    uuid = None
    try:
        uuid = str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    sampler = ClockSampler(uuid)
    if sampler:
        sampler.start()
        time.sleep(0.3)
    step_events = [new_events() for _ in range(args.steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    launches0 = gq.gptq_kernel_launches()
    t_start.record(stream)
    for k in range(args.steps):
        step(step_events[k])
    t_end.record(stream)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    launches = gq.gptq_kernel_launches() - launches0
    if sampler:
        time.sleep(0.2)
        sampler.stop()
    elapsed_ms = t_start.elapsed_time(t_end)
    stages = [[e[i].elapsed_time(e[i + 1]) for e in step_events] for i in range(nev - 1)]
    stage_ms = [statistics.mean(s) for s in stages]
    elapsed_ms = max_over_ranks(elapsed_ms, dist, dev)
    status = gq.gptq_get_device_status()
    if status != 0:
        raise RuntimeError(f"device status after the timed region: {status}")

    ms_per_step = elapsed_ms / args.steps
    value = job_rate(world, rows, n, ms_per_step)

    pk, pk_src = peaks()
    flops_syrk = float(n) * (n + 1) * spec.n_tok
    achieved = flops_syrk / (stage_ms[0] / 1e3) / 1e12
    traffic = measured_traffic(args.workload)
    # algorithmic work of the factorization (for the per-stage table)
    flops_factor = 2.0 * n ** 3 / 3.0
    result = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"{spec.name}: W {rows}x{n} {spec.w_dtype}, X {spec.n_tok} tokens x {n} bf16 "
                               f"({spec.x_kind}), {spec.bits}-bit group {spec.group}, damp {spec.damp}, "
                               f"block {spec.block}, act_order {spec.act_order}",
                   "global_batch": spec.n_tok * world, "seq_len": 2048, "parallelism": f"replicas{world}",
                   "l2": "inputs larger than L2 (X alone is %.2f GB)" % (spec.n_tok * n * 2 / 1e9),
                   "timing": "CUDA events on the launching stream; max over ranks"},
        "roofline": {"bound": "tensor", "kernel": "syrk_tc_kernel (+ its finalize kernel)", "achieved": achieved,
                     "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": achieved / pk["bf16_tflops"], "traffic": traffic,
                     "peak_source": f"{pk_src} bf16 burst (the call is timed alone with CUDA events, a few ms)",
                     "frac_of_sustained": achieved / pk["bf16_tflops_sustained"],
                     "algorithmic_flops": flops_syrk},
        "stages_ms": {"hessian": stage_ms[0], "prepare_hinv": stage_ms[1], "quantize_layer": stage_ms[2],
                      "pack": stage_ms[3]},
        "stage_rates": {"factor_tflops": flops_factor / (stage_ms[1] / 1e3) / 1e12,
                        "column_loop_weights_per_s": rows * n / (stage_ms[2] / 1e3),
                        "without_hessian_weights_per_s": rows * n / ((stage_ms[1] + stage_ms[2] + stage_ms[3]) / 1e3)},
        "gpu_launches": launches,
    }
    if sampler:
        result["clocks"] = sampler.summary()
    # a few more steps with tracing on (CUDA events around every launch):
    # per-kernel device time, outside the timed region
    trace_steps = 3
    gq.gptq_trace_read()
    gq.gptq_trace_enable(True)
    for _ in range(trace_steps):
        step(new_events())
    torch.cuda.synchronize()
    trace = gq.gptq_trace_read()
    gq.gptq_trace_enable(False)
    sm_mhz = float((result.get("clocks") or {}).get("sm_max_mhz") or 1965.0)
    result["kernel_rooflines"] = kernel_rooflines(
        trace, trace_steps, rows, n, spec.n_tok, spec.bits, ng, spec.block, pk,
        torch.cuda.get_device_properties(dev).multi_processor_count, sm_mhz)
    result["stage_rooflines"] = stage_rooflines(
        dict(zip(("hessian", "prepare_hinv", "quantize_layer", "pack"), stage_ms)), rows, n, spec.bits, ng, pk)
    result["packed_matvec"] = measure_matvec(gq, packed, out, spec, dev, pk)
    result["column_loops"] = measure_column_loops(gq, lp)
    if not args.no_gptq2d:
        cpu_rows = 64 if (world == 1 and rank == 0 and not args.no_cpu_baseline) else 0
        result["gptq2d"] = measure_gptq2d(gq, dev, result.get("clocks"), cpu_rows=cpu_rows)

    if not args.no_e2e:
        result["e2e"] = run_e2e(args, spec, W, X, dev, world, dist)

    cpu_inputs = None
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        cpu_inputs = (W[: args.cpu_rows].cpu(), X[: args.cpu_tokens].cpu())

    if world == 1 and not args.no_others:
        # every other synthetic workload once timed (outside the main timed
        # region, inputs generated on the device and freed after each)
        del lp, W, X, step, out, packed
        torch.cuda.empty_cache()
        others = {}
        for name in ("mlp_up", "mlp_down", "fc1_g128_3b", "fc2_g64_2b"):
            others[name] = measure_workload(gq, si, name, dev, steps=2, warmup=1, pk=pk,
                                            sms=torch.cuda.get_device_properties(dev).multi_processor_count,
                                            mhz=sm_mhz)
        others["layerset_block"] = measure_layerset_block(gq, si, dev, steps=2, warmup=1)
        result["other_workloads"] = others

    if cpu_inputs is not None:
        result["cpu_baseline"] = oracle_sample(cpu_inputs[0], cpu_inputs[1], spec, args.cpu_tokens, args.cpu_rows)
        for k in ("est_s_per_layer", "stage_s"):
            result["cpu_baseline"].pop(k, None)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return result if rank == 0 else None


class LayersetBlock:
    """One block of the 7B-shaped layer set (q, k, v, o; gate, up; down) on
    preallocated buffers: per input group H and U once, then the column loop
    and packing of every layer that reads that input."""

    stage_names = ("hessian", "prepare_hinv", "quantize_layer", "pack")

    def __init__(self, gq, si, dev, block_index, n_tok, bits=4, group=128, damp=0.01, block=128):
        import torch

        self.gq, self.n_tok = gq, n_tok
        self.bits, self.group, self.damp, self.block = bits, group, damp, block
        self.inputs, self.layers = si.layerset_block(block_index, n_tok=n_tok)
        self.X = {g: si.make_activations(spec, dev) for g, spec in self.inputs.items()}
        self.W = {name: si.make_weights(spec, dev) for name, spec, _ in self.layers}
        self.grp = {}
        for g, spec in self.inputs.items():
            n = spec.n
            self.grp[g] = {"H": torch.zeros((n, n), dtype=torch.float32, device=dev),
                           "U": torch.empty((n, n), dtype=torch.float32, device=dev),
                           "perm": torch.empty(n, dtype=torch.int32, device=dev),
                           "dead": torch.empty(n, dtype=torch.uint8, device=dev),
                           "ws_h": gq.workspace(gq.LIB.gptq_hessian_workspace_size(n, n_tok), dev),
                           "ws_p": gq.workspace(gq.LIB.gptq_prepare_workspace_size(n), dev)}
        self.lay = {}
        for name, spec, g in self.layers:
            rows, n = spec.rows, spec.n
            ng = gq.LIB.gptq_num_groups(n, group)
            self.lay[name] = {"g": g,
                              "out": {"codes": torch.empty((rows, n), dtype=torch.uint8, device=dev),
                                      "scales": torch.empty((rows, ng), dtype=torch.float32, device=dev),
                                      "zeros": torch.empty((rows, ng), dtype=torch.uint8, device=dev),
                                      "g_idx": torch.empty(n, dtype=torch.int32, device=dev)},
                              "packed": torch.empty((rows, gq.LIB.gptq_packed_words_per_row(n, bits)),
                                                    dtype=torch.int32, device=dev),
                              "packed_z": torch.empty((rows, gq.LIB.gptq_packed_words_per_row(ng, bits)),
                                                      dtype=torch.int32, device=dev),
                              "ws_q": gq.workspace(gq.LIB.gptq_quantize_workspace_size(rows, n, block), dev)}
        self.stream = torch.cuda.current_stream()
        self.weights = sum(spec.rows * spec.n for _, spec, _ in self.layers)

    @staticmethod
    def ev():
        import torch

        return torch.cuda.Event(enable_timing=True)

    def step(self, marks):
        gq, ev, stream = self.gq, self.ev, self.stream
        for g, b in self.grp.items():
            b["H"].zero_()
            e = [ev() for _ in range(3)]
            e[0].record(stream)
            gq.gptq_hessian_accum(b["H"], self.X[g], 2.0 / self.n_tok, ws=b["ws_h"])
            e[1].record(stream)
            gq.gptq_prepare_hinv(b["H"], self.damp, False, perm=b["perm"], dead=b["dead"], U=b["U"], ws=b["ws_p"])
            e[2].record(stream)
            marks.append(("hessian", e[0], e[1]))
            marks.append(("prepare_hinv", e[1], e[2]))
            for name, l in self.lay.items():
                if l["g"] != g:
                    continue
                f = [ev() for _ in range(3)]
                f[0].record(stream)
                gq.gptq_quantize_layer(self.W[name], b["U"], self.bits, self.group, self.block, dead=b["dead"],
                                       out=l["out"], ws=l["ws_q"])
                f[1].record(stream)
                gq.gptq_pack(l["out"]["codes"], self.bits, packed=l["packed"])
                gq.gptq_pack(l["out"]["zeros"], self.bits, packed=l["packed_z"])
                f[2].record(stream)
                marks.append(("quantize_layer", f[0], f[1]))
                marks.append(("pack", f[1], f[2]))


def measure_layerset_block(gq, si, dev, steps=2, warmup=1, n_tok=131072):
    """A few timed passes over block 0 of the layer set: per-block time,
    weights/s over the block, stage times (summed over the block's calls)."""
    import torch

    lb = LayersetBlock(gq, si, dev, 0, n_tok)
    for _ in range(warmup):
        lb.step([])
    torch.cuda.synchronize()
    marks = []
    s, e = lb.ev(), lb.ev()
    s.record(lb.stream)
    for _ in range(steps):
        lb.step(marks)
    e.record(lb.stream)
    torch.cuda.synchronize()
    ms = s.elapsed_time(e) / steps
    stage = {k: sum(a.elapsed_time(b) for s_, a, b in marks if s_ == k) / steps for k in LayersetBlock.stage_names}
    res = {"workload": f"one 7B-shaped block (q, k, v, o 4096x4096; gate, up 11008x4096; down 4096x11008; "
                       f"{lb.weights} weights), X {n_tok} tokens per input group, H and U shared by q/k/v and "
                       f"gate/up, 4-bit g128", "ms_per_block": ms, "weights_per_s": lb.weights / (ms / 1e3),
           "set_seconds_estimate": 32 * ms / 1e3, "steps": steps, "stages_ms": stage,
           "device_status": gq.gptq_get_device_status()}
    del lb
    torch.cuda.empty_cache()
    return res


def run_layerset(args, world, rank, local):
    """One block of the 7B-shaped layer set per step (replicas: rank r
    quantizes block r).  Per input group: H, U once, then every layer that
    reads that input (column loop + packing)."""
    import torch

    import post_weight_quantization_accum_b200 as gq
    import synth_inputs as si

    dist = None
    if world > 1:
        import torch.distributed as dist
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())
    n_tok = args.tokens or 131072
    lb = LayersetBlock(gq, si, dev, rank, n_tok)
    inputs, layers, stream, step, ev = lb.inputs, lb.layers, lb.stream, lb.step, lb.ev
    stage_names = LayersetBlock.stage_names

    for _ in range(args.warmup):
        step([])
    torch.cuda.synchronize()
    st = gq.gptq_get_device_status()
    if st != 0:
        raise RuntimeError(f"device status after warm-up: {st}")
    uuid = None
    try:
        uuid = str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    sampler = ClockSampler(uuid)
    if sampler:
        sampler.start()
        time.sleep(0.3)
    marks = []
    t_start, t_end = ev(), ev()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    launches0 = gq.gptq_kernel_launches()
    t_start.record(stream)
    for _ in range(args.steps):
        step(marks)
    t_end.record(stream)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    launches = gq.gptq_kernel_launches() - launches0
    if sampler:
        time.sleep(0.2)
        sampler.stop()
    ms_per_step = max_over_ranks(t_start.elapsed_time(t_end), dist, dev) / args.steps
    status = gq.gptq_get_device_status()
    if status != 0:
        raise RuntimeError(f"device status after the timed region: {status}")
    stage_ms = {k: sum(a.elapsed_time(b) for s_, a, b in marks if s_ == k) / args.steps for k in stage_names}
    weights = sum(spec.rows * spec.n for _, spec, _ in layers)
    value = world * weights / (ms_per_step / 1e3)
    pk, pk_src = peaks()
    flops_syrk = sum(float(spec.n) * (spec.n + 1) * n_tok for spec in inputs.values())
    achieved = flops_syrk / (stage_ms["hessian"] / 1e3) / 1e12
    result = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"layerset_block: one 7B-shaped block (q, k, v, o 4096x4096; gate, up 11008x4096; "
                               f"down 4096x11008; {weights} weights), X {n_tok} tokens per input group (1% outlier "
                               f"channels x20), H and U shared by q/k/v and gate/up, 4-bit g128, damp 0.01; "
                               f"the 32-block set = 32 steps",
                   "global_batch": n_tok * world, "seq_len": 2048, "parallelism": f"replicas{world}",
                   "l2": "inputs larger than L2 (6.1 GB of X per block)",
                   "timing": "CUDA events on the launching stream; max over ranks"},
        "roofline": {"bound": "tensor", "kernel": "syrk_tc_kernel (+ its finalize kernel), 4 launches per block",
                     "achieved": achieved, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": achieved / pk["bf16_tflops"], "traffic": None,
                     "peak_source": f"{pk_src} bf16 burst (each call timed alone with CUDA events)",
                     "frac_of_sustained": achieved / pk["bf16_tflops_sustained"], "algorithmic_flops": flops_syrk},
        "stages_ms": stage_ms,
        "set_seconds_estimate": 32 * ms_per_step / 1e3,
        "gpu_launches": launches,
    }
    if sampler:
        result["clocks"] = sampler.summary()
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return result if rank == 0 else None


def measure_column_loops(gq, lp, reps=10):
    """The column loop (gptq_quantize_layer on the layer's U) timed with each
    loop of gptq_set_column_loop: 0 per-block kernels (the default, the one
    the step times), 1 the fused row-slab pass; and how many codes the two
    share.  Outside the timed step."""
    import torch

    spec, st = lp.spec, lp.stream
    res = {}
    codes = {}
    try:
        for mode, name in ((0, "per_block"), (1, "fused_row_slab")):
            gq.gptq_set_column_loop(mode)

            def run():
                gq.gptq_quantize_layer(lp.W, lp.U, spec.bits, spec.group, spec.block,
                                       perm=lp.perm if spec.act_order else None, dead=lp.dead, out=lp.out, ws=lp.ws_q)

            for _ in range(3):
                run()
            torch.cuda.synchronize()
            codes[name] = lp.out["codes"].clone()
            s = torch.cuda.Event(enable_timing=True)
            e = torch.cuda.Event(enable_timing=True)
            s.record(st)
            for _ in range(reps):
                run()
            e.record(st)
            torch.cuda.synchronize()
            gq.gptq_trace_read()
            gq.gptq_trace_enable(True)
            run()
            torch.cuda.synchronize()
            trace = gq.gptq_trace_read()
            gq.gptq_trace_enable(False)
            res[name] = {"ms": s.elapsed_time(e) / reps,
                         "kernels": {k: {"launches": v[0], "ms": v[1]} for k, v in trace.items()}}
    finally:
        gq.gptq_set_column_loop(0)
    res["codes_agree"] = float((codes["per_block"] == codes["fused_row_slab"]).float().mean())
    return res


def measure_matvec(gq, packed, out, spec, dev, pk, copies=16, reps=64):
    """Inference with the layer's packed weights (batch 1, bf16 x), outside the
    timed step: per-launch time over `reps` launches that cycle through
    `copies` copies of the packed matrix (together larger than L2, so every
    launch streams its weights from HBM).  The launches are replayed from a
    CUDA graph so that the host's per-call cost does not pace them."""
    import torch

    rows, n = spec.rows, spec.n
    ng = out["scales"].shape[1]
    mats = [packed.clone() for _ in range(copies)]
    x = torch.randn(n, device=dev).to(torch.bfloat16)
    y = torch.empty((1, rows), dtype=torch.float32, device=dev)
    for i in range(3):
        gq.gptq_dequant_matvec(mats[i], out["scales"], out["zeros"], n, spec.bits, spec.group, x, y=y)
    torch.cuda.synchronize()
    gq.gptq_trace_read()  # which kernel the library dispatches for this shape
    gq.gptq_trace_enable(True)
    gq.gptq_dequant_matvec(mats[0], out["scales"], out["zeros"], n, spec.bits, spec.group, x, y=y)
    kernel = ",".join(gq.gptq_trace_read()) or "unknown"
    gq.gptq_trace_enable(False)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for i in range(reps):
            gq.gptq_dequant_matvec(mats[i % copies], out["scales"], out["zeros"], n, spec.bits, spec.group, x, y=y)
    graph.replay()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    s = torch.cuda.Event(enable_timing=True)
    e = torch.cuda.Event(enable_timing=True)
    s.record(stream)
    graph.replay()
    e.record(stream)
    torch.cuda.synchronize()
    us = s.elapsed_time(e) * 1e3 / reps
    del graph, mats
    nbytes = packed.numel() * 4 + rows * ng * 5 + n * 2 + rows * 4
    gbs = nbytes / (us * 1e-6) / 1e9
    # context: torch's bf16 matrix-vector product (a library kernel) on the
    # same shape, timed the same way (16 weight copies, graph replay)
    wb = [torch.randn((rows, n), device=dev).to(torch.bfloat16) for _ in range(copies)]
    yb = torch.empty(rows, dtype=torch.bfloat16, device=dev)
    for i in range(3):
        torch.mv(wb[i], x, out=yb)
    torch.cuda.synchronize()
    g2 = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g2):
        for i in range(reps):
            torch.mv(wb[i % copies], x, out=yb)
    g2.replay()
    torch.cuda.synchronize()
    s.record(stream)
    g2.replay()
    e.record(stream)
    torch.cuda.synchronize()
    bf16_us = s.elapsed_time(e) * 1e3 / reps
    del g2, wb
    return {"kernel": kernel, "batch": 1, "us_per_call": us,
            "torch_bf16_mv_us": bf16_us, "speedup_vs_torch_bf16_mv": bf16_us / us,
            "algorithmic_bytes": nbytes, "achieved_gbs": gbs, "peak_gbs": pk["hbm_gbs"],
            "frac": gbs / pk["hbm_gbs"], "bf16_equivalent_us_at_peak": rows * n * 2 / pk["hbm_gbs"] / 1e3}


def measure_gptq2d(gq, dev, clocks, m=4096, n=4096, tokens=8192, reps=5, cpu_rows=0):
    """GPTQ-2D (two-sided rounding) on a 4096 x 4096 matrix, outside the timed
    step: W ~ N(0, 0.02), a signed 4-bit grid (scale 0.005, codes clamped to
    [-8, 7]); HL and HR are the Grams of `tokens` N(0, 1) tokens, built and
    factored by the library (damp 0.01) before timing.  Per-call time over
    `reps` calls after 3 warm-up calls, CUDA events on the launching stream.
    Every call streams ~0.5 GB of W, factors and scratch (more than L2).
    Algorithmic work: sum over entries of (i + 1) multiply-adds for the value
    and (n - j) for the feedback row, i.e. m n (m + n) flops; the kernels are
    fp32 FMA on the CUDA cores, so the peak is SMs x 128 lanes x 2 x clock.

    With cpu_rows > 0 the fp64 oracle is timed beside it on the first cpu_rows
    rows of the same problem (an exact sample: rows i < k depend only on the
    leading k x k block of UL) and scaled by the ratio of multiply-adds."""
    import torch

    g = torch.Generator(device=dev).manual_seed(2)
    U = []
    for k in (m, n):
        X = torch.randn((tokens, k), generator=g, device=dev).to(torch.bfloat16)
        H = torch.zeros((k, k), dtype=torch.float32, device=dev)
        gq.gptq_hessian_accum(H, X, 2.0 / tokens)
        U.append(gq.gptq2d_factor(H, damp=0.01))
        del X, H
    W = 0.02 * torch.randn((m, n), generator=g, device=dev)
    codes = torch.empty((m, n), dtype=torch.int32, device=dev)
    E = torch.empty((m, n), dtype=torch.float32, device=dev)
    ws = gq.workspace(gq.LIB.gptq2d_workspace_size(m, n), dev)
    for _ in range(3):
        gq.gptq2d_round(W, U[0], U[1], 0.005, -8, 7, codes=codes, E=E, ws=ws)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    s = torch.cuda.Event(enable_timing=True)
    e = torch.cuda.Event(enable_timing=True)
    launches0 = gq.gptq_kernel_launches()
    s.record(stream)
    for _ in range(reps):
        gq.gptq2d_round(W, U[0], U[1], 0.005, -8, 7, codes=codes, E=E, ws=ws)
    e.record(stream)
    torch.cuda.synchronize()
    ms = s.elapsed_time(e) / reps
    flops = float(m) * n * (m + n)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    mhz = float((clocks or {}).get("sm_max_mhz") or 1965.0)
    peak = sms * 128 * 2 * mhz * 1e6 / 1e12
    achieved = flops / (ms * 1e-3) / 1e12
    res = {"workload": f"W {m}x{n} fp32 N(0, 0.02); HL, HR Grams of {tokens} N(0,1) tokens, damp 0.01; "
                       "scale 0.005, codes in [-8, 7]",
            "kernels": "round2d_tile_kernel (high-priority stream) + far_push_kernel (low-priority stream) per tile wavefront",
            "ms_per_call": ms, "launches_per_call": (gq.gptq_kernel_launches() - launches0) / reps,
            "weights_per_s": m * n / (ms * 1e-3),
            "roofline": {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak, "algorithmic_flops": flops,
                         "peak_source": f"fp32 FMA: {sms} SMs x 128 lanes x 2 flops x {mhz:.0f} MHz"}}
    if cpu_rows > 0:
        res["cpu_baseline"] = gptq2d_oracle_sample(W, U[0], U[1], cpu_rows)
    return res


def gptq2d_oracle_sample(W, UL, UR, k):
    """fp64 oracle on rows [0, k) of the GPTQ-2D problem, scaled to all rows by
    the ratio of multiply-adds (sum over entries of (i + 1) + (n - j))."""
    import numpy as np

    from oracle import gptq2d_oracle as g2

    m, n = W.shape
    Wh = W[:k].double().cpu().numpy()
    ULh = UL[:k, :k].double().cpu().numpy()
    URh = UR.double().cpu().numpy()
    t0 = time.perf_counter()
    g2.gptq2d(Wh, ULh, URh, 0.005, -8, 7)
    dt = time.perf_counter() - t0

    def macs(rows):
        return n * rows * (rows + 1) / 2 + rows * n * (n + 1) / 2

    scale = macs(m) / macs(k)
    est = dt * scale
    try:
        from threadpoolctl import threadpool_info
        cores = max((i.get("num_threads") or 0) for i in threadpool_info()) or len(os.sched_getaffinity(0))
    except Exception:
        cores = len(os.sched_getaffinity(0))
    return {"value": m * n / est, "unit": "weights/s", "cores": cores, "kind": "oracle",
            "sample": f"fp64 oracle on the first {k} of {m} rows (all {n} columns) of the same problem, "
                      f"measured {dt:.2f} s, scaled x{scale:.1f} by multiply-adds"}


def run_e2e(args, spec, W, X, dev, world, dist):
    """The public call with host inputs: H2D of W and X (inside the call), the
    layer pass, D2H of the packed codes, packed zero points and scales, all
    inside the timing."""
    import torch

    import post_weight_quantization_accum_b200 as gq

    Wh = W.cpu().pin_memory()
    Xh = X.cpu().pin_memory()
    stream = torch.cuda.current_stream()
    # the call allocates its own buffers through torch's caching allocator:
    # start from an empty cache and warm it (two calls) so that no timed step
    # waits on cudaMalloc / cudaFree
    torch.cuda.synchronize()
    torch.cuda.empty_cache()

    def one():
        # host inputs straight into the public call: it streams X to the GPU in
        # token chunks, each chunk's SYRK overlapping the next chunk's copy
        out = gq.quantize_layer(Wh, Xh, bits=spec.bits, group=spec.group, damp=spec.damp, block=spec.block,
                                act_order=spec.act_order, device=dev)
        res = (out["packed"].to("cpu", non_blocking=True), out["packed_zeros"].to("cpu", non_blocking=True),
               out["scales"].to("cpu", non_blocking=True))
        return res

    one()
    res = one()
    torch.cuda.synchronize()
    h2d = Wh.numel() * Wh.element_size() + Xh.numel() * Xh.element_size()
    d2h = sum(t.numel() * t.element_size() for t in res)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    s = torch.cuda.Event(enable_timing=True)
    e = torch.cuda.Event(enable_timing=True)
    s.record(stream)
    for _ in range(args.e2e_steps):
        one()
    e.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(s.elapsed_time(e) / args.e2e_steps, dist, dev)
    # the same host-to-device bytes copied alone from the same pinned buffers
    # (one copy of W and of X per step, nothing else): the link-bound floor
    Wd = torch.empty(Wh.shape, dtype=Wh.dtype, device=dev)
    Xd = torch.empty(Xh.shape, dtype=Xh.dtype, device=dev)
    torch.cuda.synchronize()
    s.record(stream)
    for _ in range(args.e2e_steps):
        Wd.copy_(Wh, non_blocking=True)
        Xd.copy_(Xh, non_blocking=True)
    e.record(stream)
    torch.cuda.synchronize()
    copy_ms = max_over_ranks(s.elapsed_time(e) / args.e2e_steps, dist, dev)
    del Wd, Xd
    return {"value": job_rate(world, spec.rows, spec.n, ms), "unit": UNIT, "ms_per_step": ms,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": args.e2e_steps,
            "h2d_only_ms": copy_ms, "h2d_only_gbs": h2d / copy_ms / 1e6,
            "frac_of_copy_bound": copy_ms / ms,
            "note": "timed region: the public call on pinned host W and X (X streamed to the GPU in token chunks "
                    "behind the SYRK) and the D2H of the packed codes, packed zero points and scales; "
                    "h2d_only_ms copies the same input bytes alone"}


# ---------------------------------------------------------------------------
# reference arm: the CPU oracle
# ---------------------------------------------------------------------------

def reference_layerset_sample():
    """fp64 oracle estimate for one block of the layer set, from a bounded
    sample: H on 2048 tokens of a 4096-wide input, the full 4096 x 4096
    factor, 16 rows of a 4096-column layer through the column loop; each
    stage scaled to every group and layer by its cost model (H ~ n^2 N,
    factor ~ n^3, column loop ~ rows n^2)."""
    import synth_inputs as si
    from oracle import gptq_oracle as go

    inputs, layers = si.layerset_block(0, n_tok=131072)
    xs = si.scaled(inputs["qkv"], n_tok=2048)
    X = si.make_activations(xs, "cpu").double().numpy()
    ws = [spec for name, spec, _ in layers if name == "q"][0]
    W = si.make_weights(ws, "cpu")[:16].double().numpy()
    t0 = time.perf_counter()
    H = go.hessian(X)
    t1 = time.perf_counter()
    prep = go.prepare(H, W, 0.01, False)
    U = go.inverse_factor(prep["H"])
    t2 = time.perf_counter()
    res = go.gptq_quantize(prep["W"], U, 4, 128, 128)
    go.pack_codes(res["codes"], 4)
    t3 = time.perf_counter()
    est = 0.0
    for spec in inputs.values():
        r = spec.n / 4096.0
        est += (t1 - t0) * r * r * (spec.n_tok / 2048.0) + (t2 - t1) * r ** 3
    for _, spec, _ in layers:
        r = spec.n / 4096.0
        est += (t3 - t2) * (spec.rows / 16.0) * r * r
    weights = sum(spec.rows * spec.n for _, spec, _ in layers)
    sample = (f"fp64 oracle: H on 2048 of 131072 tokens, the full 4096x4096 factor, 16 rows of q through the loop "
              f"(measured {t3 - t0:.2f} s), scaled to the block's 4 inputs and 7 layers (H ~ n^2 N, factor ~ n^3, "
              f"loop ~ rows n^2)")
    return weights / est, est, sample


def run_reference(args, world, rank):
    if rank != 0:
        return None
    import torch

    import synth_inputs as si

    if args.workload == "layerset_block":
        vals, ests, walls = [], [], []
        for _ in range(args.warmup + args.steps):
            t0 = time.perf_counter()
            v, est, sample = reference_layerset_sample()
            walls.append(time.perf_counter() - t0)
            vals.append(v)
            ests.append(est)
        vals, ests, walls = vals[args.warmup:], ests[args.warmup:], walls[args.warmup:]
        value = statistics.mean(vals)
        try:
            from threadpoolctl import threadpool_info
            cores = max((i.get("num_threads") or 0) for i in threadpool_info()) or len(os.sched_getaffinity(0))
        except Exception:
            cores = len(os.sched_getaffinity(0))
        cpu = {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample}
        return {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": statistics.mean(walls) * 1e3,
                "scaled_block_ms": statistics.mean(ests) * 1e3,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic",
                "config": {"workload": "layerset_block (oracle on a bounded sample, scaled to the block)",
                           "global_batch": 131072, "seq_len": 2048, "parallelism": "cpu"},
                "cpu_baseline": cpu,
                "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}

    spec = si.SPECS[args.workload]
    # a bounded sample per step (the same one the GPU arm's cpu_baseline uses)
    tokens, rows = min(args.cpu_tokens, spec.n_tok), min(args.cpu_rows, spec.rows)
    sub = si.scaled(spec, n_tok=tokens)
    W = si.make_weights(spec, "cpu")[:rows]
    X = si.make_activations(sub, "cpu")
    for _ in range(args.warmup):
        oracle_sample(W, X, spec, tokens, rows)
    vals, ests, walls, last = [], [], [], None
    for _ in range(args.steps):
        t0 = time.perf_counter()
        last = oracle_sample(W, X, spec, tokens, rows)
        walls.append(time.perf_counter() - t0)
        vals.append(last["value"])
        ests.append(last["est_s_per_layer"])
    value = statistics.mean(vals)
    cpu = {"value": value, "unit": UNIT, "cores": last["cores"], "kind": "oracle", "sample": last["sample"]}
    # ms_per_step: the sample each step actually ran; value: that sample's
    # stages scaled to the whole layer (the metric is per layer)
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": statistics.mean(walls) * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "scaled_layer_ms": statistics.mean(ests) * 1e3,
            "config": {"workload": f"{spec.name} (each step: the oracle on a bounded sample of the layer; value = "
                                   f"the sample's stages scaled to the full layer)",
                       "global_batch": spec.n_tok, "seq_len": 2048, "parallelism": "cpu"},
            "cpu_baseline": cpu,
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def profile_pass():
    """Two passes of the benchmark layer with an eighth of its tokens (the
    factorization, column loop and packing see the full shapes; X is 268 MB,
    larger than L2), then the packed-weight matvec 8 times, then one more
    pass with the fused row-slab column loop: the command that the ncu
    summaries under profiles/ capture, one kernel at a time."""
    import torch

    import post_weight_quantization_accum_b200 as gq
    import synth_inputs as si

    torch.cuda.set_device(0)
    spec = si.scaled(si.SPECS["attn4096"], n_tok=32768)
    W, X = si.make_layer(spec, "cuda")
    for _ in range(2):
        out = gq.quantize_layer(W, X, bits=spec.bits, group=spec.group, damp=spec.damp, block=spec.block)
    x = torch.randn(spec.n, device="cuda").to(torch.bfloat16)
    for _ in range(8):
        gq.gptq_dequant_matvec(out["packed"], out["scales"], out["zeros"], spec.n, spec.bits, spec.group, x)
    gq.gptq_set_column_loop(1)
    try:
        gq.quantize_layer(W, X, bits=spec.bits, group=spec.group, damp=spec.damp, block=spec.block)
    finally:
        gq.gptq_set_column_loop(0)
    torch.cuda.synchronize()
    print(json.dumps({"profile_pass": "ok", "kernel_launches": gq.gptq_kernel_launches()}))


def main():
    args = parse_args()
    if args.profile_pass:
        profile_pass()
        return
    world, rank, local = dist_env()
    if args.impl == "reference":
        res = run_reference(args, world, rank)
    elif args.workload == "layerset_block":
        res = run_layerset(args, world, rank, local)
    else:
        res = run_ours(args, world, rank, local)
    if res is not None:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
