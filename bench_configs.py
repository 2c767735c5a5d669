"""Per-workload measurements of the blockwise-FP8 (E4M3) path, for `bench.py --config 1..4`.

Each workload is one of the five configurations the benchmark is specified on (the fifth,
the full 28-layer micro-step, is bench.py's default line):

  1  one small GEMM with outlier channels: A [256, 512] (columns 17, 130, 131, 400 x50),
     W [384, 512]; quantise A (1x128) and W (128x128), then fprop. Latency-bound: the
     line's value is microseconds for the three launches.
  2  one Qwen3-1.7B-shaped block's forward linears at 4096 tokens: for QKV, O, gate/up and
     down, quantise the weight (128x128 with its transposed codes), the input (1x128), fprop.
  3  the same block's backward: for each linear, quantise dY (row-wise and along the tokens
     from one read), quantise X along the tokens, dgrad, wgrad (the weight codes of 2 are
     reused, as in training).
  4  the untied LM head at 4096 tokens: weight, hidden states (both directions), fprop
     logits, dlogits (both directions), dgrad, wgrad.

Inputs are the seeded synthetic tensors of `workloads.py` (configuration c uses seed c - 1),
resident in HBM. Every repetition first writes a 512 MB buffer and reads it back, so no
operand is left in the 126 MB L2 from the previous repetition and no dirty line is left for
the timed kernels to write back; each launch is bracketed by CUDA events on the
stream it runs on, and the median over repetitions is reported. The CPU oracle runs the
same calls (on a bounded sample for the LM head) on the host cores beside it.
"""

import json
import statistics
import time

import torch

from bench import FP8_DENSE_PEAK_TFLOPS, METRIC, Clocks, _cpu_threads, _peaks
from fp8_blockwise_scaled_e4m3_b200 import puro_fp8 as pf
from fp8_blockwise_scaled_e4m3_b200 import workloads as wl

NOMINAL_HBM_GBS = 8000.0
T4096 = 4096



def flush_l2(buf):
    """Evict the previous repetition's operands from the 126 MB L2: write a 512 MB buffer,
    then read it back, so that L2 is left holding clean lines. (After the write alone it
    would hold dirty lines, whose write-back to HBM would be charged to the next timed
    kernel.)"""
    buf.fill_(1.0)
    return buf.sum()

def _qbytes_rows(r, c):      # 1x128 row-wise: BF16 read, codes, scales
    return r * c * 3 + 4 * r * (c // 128)


def _qbytes_dual(t, c):      # both directions from one read
    return t * c * 4 + 4 * (t * (c // 128) + (t // 128) * c)


def _qbytes_cols(t, c):      # along the tokens only
    return t * c * 3 + 4 * (t // 128) * c


def _qbytes_weight(n, k, transposed=True):
    return n * k * (4 if transposed else 3) + 4 * (-(-n // 128)) * (k // 128)


class Op:
    """One library call of a workload: kind 'q' (quantiser) or 'g' (GEMM), its algorithmic
    bytes or FLOPs, and a closure that enqueues it."""

    def __init__(self, kind, name, work, fn):
        self.kind, self.name, self.work, self.fn = kind, name, work, fn


def _empty(shape, dtype, dev):
    return torch.empty(shape, dtype=dtype, device=dev)


def _weight_ops(name, w, dev, transposed=True):
    n, k = w.shape
    wq = _empty((n, k), torch.uint8, dev)
    wqt = _empty((k, n), torch.uint8, dev) if transposed else None
    ws = _empty((-(-n // 128), k // 128), torch.float32, dev)
    op = Op("q", f"{name} W 128x128", _qbytes_weight(n, k, transposed),
            lambda st: pf.puro_fp8_quantize_128x128(w, wq, wqt, ws, st))
    return op, (wq, wqt, ws)


def _rows_ops(name, x, dev):
    t, c = x.shape
    xq, xs = _empty((t, c), torch.uint8, dev), _empty((c // 128, t), torch.float32, dev)
    op = Op("q", f"{name} 1x128", _qbytes_rows(t, c), lambda st: pf.puro_fp8_quantize_1x128(x, xq, xs, st))
    return op, (xq, xs)


def _cols_ops(name, x, dev, dual):
    t, c = x.shape
    qt, st_ = _empty((c, t), torch.uint8, dev), _empty((t // 128, c), torch.float32, dev)
    q = s = None
    if dual:
        q, s = _empty((t, c), torch.uint8, dev), _empty((c // 128, t), torch.float32, dev)
    op = Op("q", f"{name} {'dual' if dual else 'along tokens'}", _qbytes_dual(t, c) if dual else _qbytes_cols(t, c),
            lambda st: pf.puro_fp8_quantize_1x128_transposed(x, qt, st_, q, s, st))
    return op, (qt, st_, q, s)


def _gemm_op(name, layout, a, a_s, b, b_s, dev):
    m, k = a.shape
    n = b.shape[0]
    c = _empty((m, n), torch.bfloat16, dev)
    lay = {"fprop": pf.PURO_FPROP, "dgrad": pf.PURO_DGRAD, "wgrad": pf.PURO_WGRAD}[layout]
    return Op("g", f"{name} {layout} {m}x{n}x{k}", 2.0 * m * n * k,
              lambda st: pf.puro_fp8_gemm_blockwise(a, a_s, b, b_s, c, lay, None, st))


def build_config(c, dev):
    """(ops, description) of workload c (1-4), inputs already on `dev`."""
    ops = []
    if c == 1:
        a, w = (t.to(dev) for t in wl.small_gemm(seed=0))
        qa, (aq, a_s) = _rows_ops("A", a, dev)
        qw, (wq, _, ws) = _weight_ops("W", w, dev, transposed=False)
        ops = [qa, qw, _gemm_op("small", "fprop", aq, a_s, wq, ws, dev)]
        return ops, "small outlier GEMM 256x384x512: quantise A (1x128), W (128x128), fprop; seed 0"
    if c in (2, 3):
        fwd = wl.layer_forward(1, T4096, dev)
        grads = wl.layer_grads(2, T4096, dev)
        for (name, x, w), (_, dy) in zip(fwd, grads):
            qw, (wq, wqt, ws) = _weight_ops(name, w, dev)
            if c == 2:
                qx, (xq, xs) = _rows_ops(f"{name} X", x, dev)
                ops += [qw, qx, _gemm_op(name, "fprop", xq, xs, wq, ws, dev)]
            else:
                qw.fn(None)  # the weight codes come from the forward; not part of this workload
                qdy, (dyqt, dyst, dyq, dys) = _cols_ops(f"{name} dY", dy, dev, dual=True)
                qx, (xqt, xst, _, _) = _cols_ops(f"{name} X", x, dev, dual=False)
                ops += [qdy, _gemm_op(name, "dgrad", dyq, dys, wqt, ws, dev), qx,
                        _gemm_op(name, "wgrad", dyqt, dyst, xqt, xst, dev)]
        what = "forward linears" if c == 2 else "backward (dgrad + wgrad) of the linears"
        return ops, f"one Qwen3-1.7B-shaped block's {what} at 4096 tokens (QKV, O, gate/up, down); seeds 1, 2"
    if c == 4:
        h, w, dl = wl.lm_head(3, T4096, dev)
        qw, (wq, wqt, ws) = _weight_ops("W_head", w, dev)
        qh, (hqt, hst, hq, hs) = _cols_ops("H", h, dev, dual=True)
        qd, (dqt, dst_, dq, ds) = _cols_ops("dlogits", dl, dev, dual=True)
        ops = [qw, qh, _gemm_op("lm_head", "fprop", hq, hs, wq, ws, dev), qd,
               _gemm_op("lm_head", "dgrad", dq, ds, wqt, ws, dev),
               _gemm_op("lm_head", "wgrad", dqt, dst_, hqt, hst, dev)]
        return ops, "untied LM head 2048 -> 151936 at 4096 tokens: fprop, dgrad, wgrad and their quantisers; seed 3"
    raise ValueError(c)


def oracle_config(c):
    """Runs workload c's calls in the CPU oracle on the host cores. Returns (GEMM FLOPs of
    the sample, seconds, sample description)."""
    import numpy as np
    from oracle import gemm as og
    from oracle import quant as oq
    bits = wl.bf16_bits
    t0 = time.perf_counter()
    flops = 0.0
    if c == 1:
        a, w = wl.small_gemm(seed=0)
        aq, a_s = oq.quant_1x128(bits(a))
        wq, _, ws = oq.quant_128x128(bits(w))
        og.gemm_ref(aq, a_s, wq, ws, "fprop")
        flops, sample = 2.0 * 256 * 384 * 512, "the whole workload"
    elif c in (2, 3):
        fwd = wl.layer_forward(1, T4096, "cpu")
        grads = wl.layer_grads(2, T4096, "cpu")
        t0 = time.perf_counter()  # input generation is not the oracle's work
        for (name, x, w), (_, dy) in zip(fwd, grads):
            wq, wqt, ws = oq.quant_128x128(bits(w))
            n, k = w.shape
            if c == 2:
                xq, xs = oq.quant_1x128(bits(x))
                og.gemm_ref(xq, xs, wq, ws, "fprop")
                flops += 2.0 * T4096 * n * k
            else:
                dyq, dys = oq.quant_1x128(bits(dy))
                dyt, dyst = oq.quant_1x128_transposed(bits(dy))
                xt, xst = oq.quant_1x128_transposed(bits(x))
                og.gemm_ref(dyq, dys, wqt, ws, "dgrad")
                og.gemm_ref(dyt, dyst, xt, xst, "wgrad")
                flops += 4.0 * T4096 * n * k
        sample = "the whole workload"
    elif c == 4:
        tok, rows = 512, 74 * 128  # a bounded sample: 512 of 4096 tokens, 74 of 1187 vocabulary blocks
        h, w, dl = wl.lm_head(3, tok, "cpu")   # timing sample only, not a parity input
        w, dl = w[:rows], dl[:, :rows].contiguous()
        t0 = time.perf_counter()
        wq, wqt, ws = oq.quant_128x128(bits(w))
        hq, hs = oq.quant_1x128(bits(h))
        og.gemm_ref(hq, hs, wq, ws, "fprop")
        dq, ds = oq.quant_1x128(bits(dl))
        dt_, dst_ = oq.quant_1x128_transposed(bits(dl))
        ht, hst = oq.quant_1x128_transposed(bits(h))
        og.gemm_ref(dq, ds, wqt, ws, "dgrad")
        og.gemm_ref(dt_, dst_, ht, hst, "wgrad")
        flops = 6.0 * tok * rows * 2048
        sample = f"{tok} of 4096 tokens x {rows} of 151936 vocabulary rows, all six calls"
    else:
        raise ValueError(c)
    return flops, time.perf_counter() - t0, sample


def run_config(c, args):
    dev = torch.device("cuda", torch.cuda.current_device())
    hbm_gbs, bf16_tf, bf16_tf_sus, peak_src = _peaks()
    fp8_burst = 2.0 * bf16_tf   # isolated kernels: the burst figure, x2 for FP8 (nominal ratio)
    ops, desc = build_config(c, dev)
    stream = torch.cuda.current_stream()
    flush = torch.empty(512 * 2 ** 20 // 4, dtype=torch.float32, device=dev)
    torch.cuda.synchronize()
    per_op = [[] for _ in ops]
    whole = []
    clocks = Clocks(torch.cuda.current_device())
    clocks.start()
    t_begin = None
    for rep in range(args.warmup + args.reps):
        if rep == args.warmup:
            pf.puro_fp8_sync_status()
            t_begin = time.time()
        flush_l2(flush)
        evs = [torch.cuda.Event(enable_timing=True)]
        evs[0].record(stream)
        for op in ops:
            op.fn(stream)
            e = torch.cuda.Event(enable_timing=True)
            e.record(stream)
            evs.append(e)
        evs[-1].synchronize()
        if rep >= args.warmup:
            for i in range(len(ops)):
                per_op[i].append(evs[i].elapsed_time(evs[i + 1]))
            whole.append(evs[0].elapsed_time(evs[-1]))
    clk = clocks.stop(t_begin, time.time())
    pf.puro_fp8_sync_status()
    med = [statistics.median(t) for t in per_op]
    ms_whole = statistics.median(whole)
    g_flops = sum(op.work for op in ops if op.kind == "g")
    q_bytes = sum(op.work for op in ops if op.kind == "q")
    g_ms = sum(m for m, op in zip(med, ops) if op.kind == "g")
    q_ms = sum(m for m, op in zip(med, ops) if op.kind == "q")
    g_tf = g_flops / (g_ms * 1e-3) / 1e12
    q_gbs = q_bytes / (q_ms * 1e-3) / 1e9
    line = {"metric": METRIC, "n_gpus": 1, "steps": args.reps, "warmup": args.warmup,
            "dtype": "e4m3", "data": "synthetic", "scaling": "weak", "vs_baseline": None,
            "config": {"workload": desc, "config_index": c,
                       "l2": "flushed before every repetition (512 MB written, then read back)"},
            "ms_per_step": round(ms_whole, 4), "gpu_launches": len(ops) * args.reps, "clocks": clk}
    if c == 1:
        line.update({"value": round(ms_whole * 1e3, 2), "unit": "us", "higher_is_better": False,
                     "note": "latency-bound (6 output tiles on 148 SMs); TFLOP/s is context only",
                     "gemm_tflops": round(g_tf, 2)})
    else:
        line.update({"value": round(g_flops / (ms_whole * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
                     "higher_is_better": True})
    line["roofline"] = {"bound": "tensor", "kernel": "k_gemm_blockwise", "achieved": round(g_tf, 1),
                        "peak": round(fp8_burst, 1), "unit": "TFLOP/s", "frac": round(g_tf / fp8_burst, 4),
                        "frac_of_nominal_4500": round(g_tf / FP8_DENSE_PEAK_TFLOPS, 4),
                        "peak_note": f"2 x {peak_src} burst BF16 ({bf16_tf})", "traffic": None}
    line["roofline_quant"] = {"bound": "hbm", "kernel": "k_quant_tiles", "achieved": round(q_gbs, 1),
                              "peak": hbm_gbs, "unit": "GB/s", "frac": round(q_gbs / hbm_gbs, 4),
                              "frac_of_nominal_8000": round(q_gbs / NOMINAL_HBM_GBS, 4),
                              "peak_note": f"{peak_src} copy bandwidth"}
    line["ops"] = [{"op": op.name, "us": round(m * 1e3, 2),
                    ("tflops" if op.kind == "g" else "gbs"): round(op.work / (m * 1e-3) / (1e12 if op.kind == "g" else 1e9), 1)}
                   for m, op in zip(med, ops)]
    if not args.no_cpu_baseline:
        flops, secs, sample = oracle_config(c)
        cb = {"kind": "oracle", "cores": _cpu_threads(), "sample": sample, "seconds": round(secs, 3)}
        if c == 1:
            cb.update({"value": round(secs * 1e6, 1), "unit": "us"})
        else:
            cb.update({"value": round(flops / secs / 1e12, 6), "unit": "TFLOP/s"})
        line["cpu_baseline"] = cb
    print(json.dumps(line), flush=True)
    del ops, flush
    torch.cuda.empty_cache()


def run_fused_comparison(args):
    """fprop and dgrad of one Qwen3-1.7B-shaped block at 8192 tokens, each timed two ways:
    the GEMM followed by a separate 1x128 quantisation of its BF16 output (the input of the
    next linear), and puro_fp8_gemm_blockwise_quant, which writes both from one launch.
    Same operands, L2 flushed before every repetition, median over repetitions."""
    dev = torch.device("cuda", torch.cuda.current_device())
    T = 8192
    fwd = wl.layer_forward(4, T, dev, layer=0)
    grads = wl.layer_grads(4, T, dev, layer=0)
    flush = torch.empty(512 * 2 ** 20 // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    cases = []
    for (name, x, w), (_, dy) in zip(fwd, grads):
        xq, xs = pf.quantize_1x128(x)
        wq, wqt, ws = pf.quantize_128x128(w)
        dyq, dys = pf.quantize_1x128(dy)
        cases.append((f"{name} fprop", "fprop", (xq, xs, wq, ws)))
        cases.append((f"{name} dgrad", "dgrad", (dyq, dys, wqt, ws)))
    rows = []
    for label, layout, ops in cases:
        m, n = ops[0].shape[0], ops[2].shape[0]
        c = torch.empty((m, n), dtype=torch.bfloat16, device=dev)
        cq = torch.empty((m, n), dtype=torch.uint8, device=dev)
        cs = torch.empty((n // 128, m), dtype=torch.float32, device=dev)
        lay = {"fprop": pf.PURO_FPROP, "dgrad": pf.PURO_DGRAD}[layout]

        def separate(st):
            pf.puro_fp8_gemm_blockwise(*ops, c, lay, None, st)
            pf.puro_fp8_quantize_1x128(c, cq, cs, st)

        def fused(st):
            pf.puro_fp8_gemm_blockwise_quant(*ops, c, cq, cs, lay, st)

        t = {"separate": [], "fused": []}
        for rep in range(args.warmup + args.reps):
            for kind, fn in (("separate", separate), ("fused", fused)):
                flush_l2(flush)
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                fn(stream)
                e1.record(stream)
                e1.synchronize()
                if rep >= args.warmup:
                    t[kind].append(e0.elapsed_time(e1))
        sep, fus = statistics.median(t["separate"]), statistics.median(t["fused"])
        rows.append({"op": label, "M": m, "N": n, "K": ops[0].shape[1], "separate_us": round(sep * 1e3, 1),
                     "fused_us": round(fus * 1e3, 1), "saved_pct": round(100 * (1 - fus / sep), 1)})
        del c, cq, cs
    pf.puro_fp8_sync_status()
    tot_sep = sum(r["separate_us"] for r in rows)
    tot_fus = sum(r["fused_us"] for r in rows)
    print(json.dumps({"comparison": "GEMM + separate 1x128 quantiser of its output vs the fused epilogue",
                      "workload": "fprop and dgrad of one Qwen3-1.7B-shaped block at 8192 tokens, seed 4",
                      "l2": "flushed before every repetition (512 MB written, then read back)", "reps": args.reps,
                      "total_separate_us": round(tot_sep, 1), "total_fused_us": round(tot_fus, 1),
                      "saved_pct": round(100 * (1 - tot_fus / tot_sep), 1), "ops": rows}), flush=True)


def run_grouped_comparison(args):
    """The four weight gradients of one Qwen3-1.7B-shaped block at 8192 tokens: four
    puro_fp8_gemm_blockwise launches against one puro_fp8_gemm_blockwise_grouped launch.
    Same operands, L2 flushed before every repetition, median over repetitions."""
    dev = torch.device("cuda", torch.cuda.current_device())
    T = 8192
    fwd = wl.layer_forward(4, T, dev, layer=0)
    grads = wl.layer_grads(4, T, dev, layer=0)
    problems = []
    flops = 0.0
    for (name, x, w), (_, dy) in zip(fwd, grads):
        dyt, dyst = pf.quantize_1x128_transposed(dy)
        xt, xst = pf.quantize_1x128_transposed(x)
        problems.append((dyt, dyst, xt, xst, torch.empty(w.shape, dtype=torch.bfloat16, device=dev)))
        flops += 2.0 * w.shape[0] * w.shape[1] * T
    flush = torch.empty(512 * 2 ** 20 // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    def separate(st):
        for pr in problems:
            pf.puro_fp8_gemm_blockwise(*pr, pf.PURO_WGRAD, None, st)

    def grouped(st):
        pf.puro_fp8_gemm_blockwise_grouped(problems, pf.PURO_WGRAD, st)

    t = {"separate": [], "grouped": []}
    for rep in range(args.warmup + args.reps):
        for kind, fn in (("separate", separate), ("grouped", grouped)):
            flush_l2(flush)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn(stream)
            e1.record(stream)
            e1.synchronize()
            if rep >= args.warmup:
                t[kind].append(e0.elapsed_time(e1))
    pf.puro_fp8_sync_status()
    sep, grp = statistics.median(t["separate"]), statistics.median(t["grouped"])
    print(json.dumps({"comparison": "four wgrad launches vs one grouped launch",
                      "workload": "wgrads of one Qwen3-1.7B-shaped block (QKV, O, gate/up, down) at 8192 tokens, seed 4",
                      "l2": "flushed before every repetition (512 MB written, then read back)", "reps": args.reps,
                      "separate_us": round(sep * 1e3, 1), "grouped_us": round(grp * 1e3, 1),
                      "separate_tflops": round(flops / sep / 1e9, 1), "grouped_tflops": round(flops / grp / 1e9, 1),
                      "saved_pct": round(100 * (1 - grp / sep), 1)}), flush=True)


def run_scales_comparison(args):
    """The full micro-step (28 Qwen3-1.7B-shaped layers and the LM head at 8192 tokens,
    fprop + dgrad + wgrad) in both scale modes, one after the other on the same seeded
    inputs: the method's FP32 scales (amax / 448) with the blockwise GEMM, and power-of-two
    UE8M0 scales with the block-scaled GEMM. Each mode: args.warmup untimed steps, then
    `steps` steps between two CUDA events (inputs larger than L2), then one pass with an
    event after every launch for the GEMM / quantiser split."""
    from bench import Step
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream()
    steps = max(1, min(args.steps, 10))
    out = {}
    for mode in ("fp32", "pow2"):
        step = Step(pf, wl, args.tokens, args.layers, dev, seed=4, scales=mode, lm_head=not args.no_lm_head)
        for _ in range(args.warmup):
            step.run(stream=stream, overlap=True)
        pf.puro_fp8_sync_status()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            step.run(stream=stream, overlap=True)
        e1.record(stream)
        e1.synchronize()
        ms = e0.elapsed_time(e1) / steps
        events = [("start", torch.cuda.Event(enable_timing=True))]
        events[0][1].record(stream)
        step.run(ev=events, stream=stream)
        events[-1][1].synchronize()
        pf.puro_fp8_sync_status()
        t = {"g": 0.0, "q": 0.0}
        for (_, a), (kind, b) in zip(events[:-1], events[1:]):
            t[kind] += a.elapsed_time(b)
        out[mode] = {"ms_per_step": round(ms, 3), "tflops": round(step.gemm_flops / (ms * 1e-3) / 1e12, 1),
                     "gemm_ms": round(t["g"], 3), "gemm_tflops": round(step.gemm_flops / (t["g"] * 1e-3) / 1e12, 1),
                     "quant_ms": round(t["q"], 3), "quant_gbs": round(step.quant_bytes / (t["q"] * 1e-3) / 1e9, 1),
                     "launches": step.launches_per_step}
        del step
        torch.cuda.empty_cache()
    print(json.dumps({"comparison": "full step, FP32 scales + blockwise GEMM vs power-of-two scales + "
                                    "block-scaled GEMM",
                      "workload": f"qwen3-1.7b-linear-stack-{args.layers}L"
                                  f"{'' if args.no_lm_head else '+lm_head'} fwd+dgrad+wgrad, "
                                  f"{args.tokens} tokens, seed 4",
                      "steps": steps, "warmup": args.warmup, **out,
                      "pow2_speedup": round(out["fp32"]["ms_per_step"] / out["pow2"]["ms_per_step"], 3)}),
          flush=True)


def run_vendor_reference(args):
    """Context for the GEMM roofline, not part of the path: the library FP8 GEMM
    (torch._scaled_mm, per-tensor scales, BF16 output, no blockwise scaling) and the BF16 GEMM
    on the step's GEMM shapes, back to back with CUDA events. What a plain FP8 GEMM reaches on
    this GPU bounds what a blockwise one can."""
    dev = torch.device("cuda", torch.cuda.current_device())
    T = args.tokens
    shapes = [("fprop QKV", T, 4096, 2048), ("fprop gate/up", T, 12288, 2048), ("fprop down", T, 2048, 6144),
              ("dgrad gate/up", T, 2048, 12288), ("wgrad gate/up", 12288, 2048, T), ("square", 8192, 8192, 8192)]
    g = torch.Generator(device=dev)
    g.manual_seed(0)
    rows = []
    for label, M, N, K in shapes:
        a = torch.randn(M, K, device=dev, generator=g).to(torch.float8_e4m3fn)
        b = torch.randn(N, K, device=dev, generator=g).to(torch.float8_e4m3fn)
        one = torch.ones((), device=dev)
        fns = {"fp8": lambda: torch._scaled_mm(a, b.t(), scale_a=one, scale_b=one, out_dtype=torch.bfloat16)}
        a16, b16 = a.to(torch.bfloat16), b.to(torch.bfloat16)
        fns["bf16"] = lambda: a16 @ b16.t()
        row = {"op": label, "M": M, "N": N, "K": K}
        for kind, fn in fns.items():
            for _ in range(3):
                fn()
            torch.cuda.synchronize()
            t = []
            for _ in range(max(3, args.reps // 2)):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                for _ in range(10):
                    fn()
                e1.record()
                e1.synchronize()
                t.append(e0.elapsed_time(e1) / 10)
            row[f"{kind}_tflops"] = round(2.0 * M * N * K / statistics.median(t) / 1e9, 1)
        rows.append(row)
        del a, b, a16, b16
    print(json.dumps({"reference": "library GEMMs (torch._scaled_mm FP8 with per-tensor scales; BF16 matmul)",
                      "note": "context for the roofline only; not on the path", "ops": rows}), flush=True)


def run_kernel_comparison(args):
    """Single GEMMs at the step's shapes (8192 tokens), each with FP32 scales
    (puro_fp8_gemm_blockwise) and with power-of-two scales (puro_fp8_mx_gemm) on the same
    random codes (the scale bytes 2^(byte - 127) as the FP32 scales), back to back with CUDA
    events, interleaved, median over repetitions."""
    dev = torch.device("cuda", torch.cuda.current_device())
    T = args.tokens
    shapes = [("fprop", T, 4096, 2048), ("fprop", T, 12288, 2048), ("fprop", T, 2048, 6144),
              ("dgrad", T, 2048, 12288), ("dgrad", T, 2048, 4096), ("wgrad", 12288, 2048, T),
              ("wgrad", 4096, 2048, T), ("wgrad", 2048, 6144, T), ("fprop", T, 151936, 2048)]
    g = torch.Generator(device=dev)
    g.manual_seed(0)
    rows = []
    for lay, M, N, K in shapes:
        aq = torch.randint(0, 256, (M, K), dtype=torch.uint8, device=dev, generator=g)
        bq = torch.randint(0, 256, (N, K), dtype=torch.uint8, device=dev, generator=g)
        for t in (aq, bq):
            t[(t & 0x7F) == 0x7F] = 0x38  # no NaN codes
        nb = (N + 127) // 128
        bs_shape = {"fprop": (nb, K // 128), "dgrad": (K // 128, nb), "wgrad": (K // 128, N)}[lay]
        ab = torch.randint(112, 124, (K // 128, M), dtype=torch.uint8, device=dev, generator=g)
        bb = torch.randint(112, 124, bs_shape, dtype=torch.uint8, device=dev, generator=g)
        a_s, b_s = torch.exp2(ab.float() - 127), torch.exp2(bb.float() - 127)
        c32 = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        cmx = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        fns = {"fp32_scales": lambda: pf.puro_fp8_gemm_blockwise(aq, a_s, bq, b_s, c32, lay),
               "pow2_scales": lambda: pf.puro_fp8_mx_gemm(aq, ab, bq, bb, cmx, lay)}
        for fn in fns.values():
            fn()
            fn()
        torch.cuda.synchronize()
        t = {k: [] for k in fns}
        for _ in range(max(3, args.reps // 2)):
            for k, fn in fns.items():
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                for _ in range(5):
                    fn()
                e1.record()
                e1.synchronize()
                t[k].append(e0.elapsed_time(e1) / 5)
        pf.puro_fp8_sync_status()
        flops = 2.0 * M * N * K
        rows.append({"op": lay, "M": M, "N": N, "K": K,
                     **{f"{k}_tflops": round(flops / statistics.median(v) / 1e9, 1) for k, v in t.items()}})
        del aq, bq, ab, bb, a_s, b_s, c32, cmx
    print(json.dumps({"comparison": "single GEMMs at the step's shapes: FP32 scales vs power-of-two scales",
                      "inputs": "random E4M3 codes, scale bytes 112..123 (the same scales as FP32 for the other kernel)",
                      "ops": rows}), flush=True)


NVFP4_BYTES_PER_ELEMENT = 2 + 2 + 0.5 + 1 / 16  # amax read, quantise read, codes, factors
NVFP4_DUAL_BYTES_PER_ELEMENT = 2 + 2 + 2 * (0.5 + 1 / 16)  # the same, both layouts from one read


def run_nvfp4(args):
    """The NVFP4 mode on the step's shapes (8192 tokens), CUDA events, L2 flushed before every
    timed call (512 MB written and read back), median over repetitions:
    - the 1x16 quantisers (row-wise, along the tokens written transposed, and both from one
      call) on the step's activation, gradient and weight shapes, in GB/s of algorithmic bytes:
      the tensor-amax pass reads X once, the quantising pass reads it again and writes the
      packed codes and one factor byte per 16 elements (4.5625 bytes per element; 5.125 for
      both layouts);
    - the GEMMs of the kernel comparison (fprop, dgrad, wgrad and LM-head shapes), each on
      operands the NVFP4 quantisers made from seeded random BF16 tensors, in TFLOP/s and as
      a fraction of the dense FP4 tensor peak, taken as 4 x the BF16 peak (the nominal ratio
      of the dense FP4 and BF16 rates)."""
    dev = torch.device("cuda", torch.cuda.current_device())
    T = args.tokens
    _, bf16_tf, _, peak_src = _peaks()
    fp4_peak = 4.0 * bf16_tf
    flush = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    reps = max(3, args.reps // 2)

    def timed(fn):
        fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(reps):
            flush_l2(flush)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            e1.synchronize()
            ts.append(e0.elapsed_time(e1))
        pf.puro_fp8_sync_status()
        return statistics.median(ts)

    def rand(shape, seed):
        g = torch.Generator(device=dev)
        g.manual_seed(seed)
        return torch.randn(shape, generator=g, device=dev).to(torch.bfloat16)

    quant = []
    for name, r, c, mode in (("X 1x16", T, 2048, "rows"), ("X along tokens", T, 2048, "cols"),
                             ("X both (dual)", T, 2048, "dual"), ("X 1x16", T, 6144, "rows"),
                             ("X both (dual)", T, 6144, "dual"), ("dY 1x16", T, 12288, "rows"),
                             ("dY along tokens", T, 12288, "cols"), ("dY both (dual)", T, 12288, "dual"),
                             ("W gate/up 1x16", 12288, 2048, "rows"), ("W gate/up along N_out", 12288, 2048, "cols"),
                             ("W gate/up both (dual)", 12288, 2048, "dual"),
                             ("LM-head dY both (dual)", T, 151936, "dual")):
        x = rand((r, c), 7 + len(quant))
        amax = torch.empty(1, dtype=torch.float32, device=dev)
        q = torch.empty((r, c // 2), dtype=torch.uint8, device=dev)
        f = torch.empty(((c + 255) // 256, r, 16), dtype=torch.uint8, device=dev)
        qt = torch.empty((c, r // 2), dtype=torch.uint8, device=dev)
        ft = torch.empty(((r + 255) // 256, c, 16), dtype=torch.uint8, device=dev)
        fn = {"rows": lambda: pf.puro_nvfp4_quantize_1x16(x, q, f, amax),
              "cols": lambda: pf.puro_nvfp4_quantize_1x16_transposed(x, qt, ft, amax),
              "dual": lambda: pf.puro_nvfp4_quantize_1x16_dual(x, q, f, qt, ft, amax)}[mode]
        ms = timed(fn)
        gb = r * c * (NVFP4_DUAL_BYTES_PER_ELEMENT if mode == "dual" else NVFP4_BYTES_PER_ELEMENT) / 1e9
        quant.append({"tensor": name, "R": r, "C": c, "us": round(ms * 1e3, 1), "GB_per_s": round(gb / (ms * 1e-3), 1)})
        del x, q, f, qt, ft
        torch.cuda.empty_cache()

    shapes = [("fprop", T, 4096, 2048), ("fprop", T, 12288, 2048), ("fprop", T, 2048, 6144),
              ("dgrad", T, 2048, 12288), ("dgrad", T, 2048, 4096), ("wgrad", 12288, 2048, T),
              ("wgrad", 4096, 2048, T), ("wgrad", 2048, 6144, T), ("fprop", T, 151936, 2048)]
    gemms = []
    for i, (lay, M, N, K) in enumerate(shapes):
        aq, af, aa = pf.nvfp4_quantize(rand((M, K), 100 + i))
        b = rand((N, K), 200 + i)
        bq, bf, ba = pf.nvfp4_quantize(b)
        del b
        c = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        ms = timed(lambda: pf.puro_nvfp4_gemm(aq, af, aa, bq, bf, ba, c))
        tf = 2.0 * M * N * K / (ms * 1e-3) / 1e12
        gemms.append({"op": lay, "M": M, "N": N, "K": K, "us": round(ms * 1e3, 1), "tflops": round(tf, 1),
                      "frac_of_fp4_peak": round(tf / fp4_peak, 4)})
        del aq, af, bq, bf, c
        torch.cuda.empty_cache()
    print(json.dumps({"comparison": "NVFP4 (E2M1, UE4M3 per 16, FP32 tensor scale): quantisers and GEMMs",
                      "workload": f"the Qwen3-1.7B-shaped step's tensors at {T} tokens, seeded random BF16",
                      "l2": "flushed before every timed call (512 MB written, then read back)",
                      "fp4_peak_tflops": round(fp4_peak, 1),
                      "fp4_peak_note": f"4 x {peak_src} BF16 burst ({bf16_tf}) (dense FP4 / BF16 nominal ratio)",
                      "quant_bytes_per_element": NVFP4_BYTES_PER_ELEMENT,
                      "dual_bytes_per_element": NVFP4_DUAL_BYTES_PER_ELEMENT, "quantisers": quant, "gemms": gemms}),
          flush=True)


def run_nvfp4_step(args):
    """The full micro-step (28 Qwen3-1.7B-shaped layers and the LM head at 8192 tokens, fprop +
    dgrad + wgrad) in NVFP4 against the method's FP32-scale step, on the same seeded inputs in
    one process. NVFP4 needs each of W, X and dY in two layouts: W row-wise (fprop) and along
    N_out (dgrad), X row-wise and along the tokens, dY row-wise and along the tokens. Timed two
    ways: with the single-layout quantisers (two calls per tensor, each an amax launch and a
    codes launch: 15 launches per linear with the three GEMMs), and with the dual quantiser
    (one call per tensor: 9 launches per linear). Every variant runs on one stream, captured
    once into a CUDA graph and replayed; args.warmup replays, then `steps` replays between two
    CUDA events (inputs larger than L2). The FP32-scale step is also timed as bench.py's
    default runs it (weight quantisers and wgrads on a second stream)."""
    from bench import Step
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.Stream(device=dev)
    torch.cuda.set_stream(stream)
    steps = max(1, min(args.steps, 10))
    step = Step(pf, wl, args.tokens, args.layers, dev, seed=4, lm_head=not args.no_lm_head)
    T = args.tokens
    u8 = torch.uint8

    def both(r, c):
        """(row-wise codes, factors, amax), (transposed codes, factors, amax) buffers of [r, c]."""
        return ((torch.empty((r, c // 2), dtype=u8, device=dev), torch.empty(((c + 255) // 256, r, 16), dtype=u8, device=dev),
                 torch.empty(1, dtype=torch.float32, device=dev)),
                (torch.empty((c, r // 2), dtype=u8, device=dev), torch.empty(((r + 255) // 256, c, 16), dtype=u8, device=dev),
                 torch.empty(1, dtype=torch.float32, device=dev)))

    lin_bufs, shape_bufs = [], {}
    for _, x, w, dy, *_ in step.linears:
        n, k = w.shape
        wr, wt = both(n, k)
        lin_bufs.append({"w": wr, "wt": wt, "xt": both(T, k)[1]})
        if (n, k) not in shape_bufs:
            dyr, dyt = both(T, n)
            shape_bufs[(n, k)] = {"x": both(T, k)[0], "dy": dyr, "dyt": dyt,
                                  "y": torch.empty((T, n), dtype=torch.bfloat16, device=dev),
                                  "dx": torch.empty((T, k), dtype=torch.bfloat16, device=dev),
                                  "dw": torch.empty((n, k), dtype=torch.bfloat16, device=dev)}

    def quantise_both(t, rows, cols, dual):
        """rows = (q, f, amax), cols = (qt, ft, amax'); with `dual` one call fills both and writes
        the tensor's amax into cols (X's row-wise buffers are shared by the linears of one shape
        while its transposed ones are kept per linear until its wgrad)."""
        if dual:
            pf.puro_nvfp4_quantize_1x16_dual(t, rows[0], rows[1], cols[0], cols[1], cols[2])
        else:
            pf.puro_nvfp4_quantize_1x16(t, *rows)
            pf.puro_nvfp4_quantize_1x16_transposed(t, *cols)

    def nv_step(dual):
        g = pf.puro_nvfp4_gemm
        ar = (lambda rows, cols: cols[2]) if dual else (lambda rows, cols: rows[2])  # row-wise side's amax
        for (_, x, w, dy, *_), lb in zip(step.linears, lin_bufs):
            quantise_both(w, lb["w"], lb["wt"], dual)
        for (_, x, w, dy, *_), lb in zip(step.linears, lin_bufs):
            sb = shape_bufs[tuple(w.shape)]
            quantise_both(x, sb["x"], lb["xt"], dual)
            g(*sb["x"][:2], ar(sb["x"], lb["xt"]), *lb["w"][:2], ar(lb["w"], lb["wt"]), sb["y"])
        for i in range(len(step.linears) - 1, -1, -1):
            _, x, w, dy, *_ = step.linears[i]
            lb, sb = lin_bufs[i], shape_bufs[tuple(w.shape)]
            quantise_both(dy, sb["dy"], sb["dyt"], dual)
            g(*sb["dy"][:2], ar(sb["dy"], sb["dyt"]), *lb["wt"], sb["dx"])
            g(*sb["dyt"], *lb["xt"], sb["dw"])

    def timed_graph(fn):
        for _ in range(2):
            fn()
        torch.cuda.synchronize()
        pf.puro_fp8_sync_status()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            fn()
        for _ in range(max(1, args.warmup)):
            graph.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            graph.replay()
        e1.record(stream)
        e1.synchronize()
        pf.puro_fp8_sync_status()
        del graph
        return e0.elapsed_time(e1) / steps

    out = {}
    for name, fn in (("fp32_scales_one_stream", lambda: step.run(stream=stream, overlap=False)),
                     ("fp32_scales_two_streams", lambda: step.run(stream=stream, overlap=True)),
                     ("nvfp4_single_layout_quantisers", lambda: nv_step(False)),
                     ("nvfp4_dual_quantiser", lambda: nv_step(True))):
        ms = timed_graph(fn)
        out[name] = {"ms_per_step": round(ms, 3), "tflops": round(step.gemm_flops / (ms * 1e-3) / 1e12, 1)}
    n_lin = len(step.linears)
    out["launches"] = {"nvfp4_single_layout_quantisers": 15 * n_lin, "nvfp4_dual_quantiser": 9 * n_lin}
    out["nvfp4_dual_speedup_vs_fp32_scales_one_stream"] = round(
        out["fp32_scales_one_stream"]["ms_per_step"] / out["nvfp4_dual_quantiser"]["ms_per_step"], 3)
    print(json.dumps({"comparison": "full step: FP32 scales + blockwise FP8 GEMM vs NVFP4 quantisers + FP4 GEMM",
                      "workload": f"qwen3-1.7b-linear-stack-{args.layers}L{'' if args.no_lm_head else '+lm_head'} "
                                  f"fwd+dgrad+wgrad, {T} tokens, seed 4",
                      "steps": steps, "warmup": args.warmup, **out}), flush=True)
