#!/usr/bin/env python
"""Benchmark of the blockwise-FP8 (E4M3) linear path on B200.

One step = every quantise and GEMM call of one training micro-step of a
Qwen3-1.7B-shaped model with an untied LM head (28 blocks of QKV, O, gate/up and down
linears plus the 151936-wide head) over one micro-batch of 2 x 4096 = 8192 tokens:
  weights:        quantise every W (128x128, with the transposed codes)
  forward sweep  (blocks 0..27, head):  quantise X (1x128 row-wise for fprop and along
                                        the tokens for wgrad, one read), fprop GEMM
  backward sweep (head, blocks 27..0):  quantise dY (row-wise + along the tokens, one
                                        read), dgrad and wgrad
That is 6 launches per linear, 678 per step, 84.56 TFLOP of GEMM work (2MNK, i.e.
6 x linear parameters x tokens) and 42.5 GB of quantiser traffic. Inputs are seeded
synthetic BF16 tensors resident in HBM (about 21 GB, distinct per block, so every step
reads far more than the 126 MB L2).

Printed (rank 0): one JSON line. `value` is GEMM TFLOP/s of the whole step (quantisers
included in the time), summed over ranks; `roofline` is the GEMM kernel alone (CUDA
events around every launch, in a separate pass of up to 5 steps after the timed region)
against the tensor peak; `roofline_quant`
the quantisers against HBM bandwidth; `cpu_baseline` the CPU oracle on a bounded
sample; `e2e` the same step through the public API with the inputs copied from pinned
host memory and the weight gradients copied back, inside the timed region.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
Multi-GPU: launch with torchrun; each rank runs its own micro-batch (weak scaling, no
collective in the data path; the timing is the max over ranks).
"""

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import tempfile
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "FP8 blockwise GEMM TFLOP/s (fwd+dgrad+wgrad, Qwen3-1.7B shapes) and % FP8 peak"
FP8_DENSE_PEAK_TFLOPS = 4500.0  # nominal B200 dense FP8
WORKLOAD = "qwen3-1.7b-linear-stack-28L+lm_head fwd+dgrad+wgrad, 8192 tokens (2x4096)"


def workload_name(args):
    """WORKLOAD for the default sizes; the same form for a reduced (profiling) step."""
    if args.layers == 28 and args.tokens == 8192 and not args.no_lm_head:
        return WORKLOAD
    head = "" if args.no_lm_head else "+lm_head"
    return f"qwen3-1.7b-linear-stack-{args.layers}L{head} fwd+dgrad+wgrad, {args.tokens} tokens"


def _args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--tokens", type=int, default=8192)
    p.add_argument("--layers", type=int, default=28)
    p.add_argument("--e2e-steps", type=int, default=3)
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-graph", action="store_true",
                   help="issue the timed steps' launches one by one instead of replaying a CUDA graph")
    p.add_argument("--no-lm-head", action="store_true",
                   help="leave the LM head out of the step (small profiling cases with --layers)")
    p.add_argument("--no-group", action="store_true",
                   help="one wgrad launch per linear instead of one grouped launch per block")
    p.add_argument("--config", default="5",
                   help="workload: 1 small outlier GEMM, 2 one layer's forward linears, 3 its backward, "
                        "4 the LM head, 5 the full 28-layer step (default), 'all' for 1-4 then 5, or "
                        "'fused' for the fused epilogue quantisation against GEMM + separate quantiser, "
                        "'grouped' for one block's four wgrads in one launch against four, "
                        "'scales' for the full step with FP32 scales against power-of-two scales, "
                        "'vendor' for the library FP8 and BF16 GEMMs on the step's shapes (roofline context), "
                        "'kernels' for single GEMMs with FP32 against power-of-two scales, "
                        "'nvfp4' for the NVFP4 quantisers and GEMMs on the step's shapes, "
                        "'nvfp4-step' for the whole step in NVFP4 against FP32 scales")
    p.add_argument("--reps", type=int, default=10, help="timed repetitions of configs 1-4")
    return p.parse_args()


FALLBACK_PEAKS = (6650.0, 1590.0, 1400.0)  # HBM GB/s, BF16 TFLOP/s burst, BF16 TFLOP/s sustained


def _peaks(path=None):
    """(HBM GB/s, BF16 TFLOP/s burst, BF16 TFLOP/s sustained, source) from the measured-peaks file
    when it is there and readable (a value may also be an object holding "value"), else the
    fallback figures."""
    path = path or os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        try:
            with open(path) as f:
                d = json.load(f)
            vals = []
            for key in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained"):
                v = d[key]
                if isinstance(v, dict):
                    v = v["value"]
                v = float(v)
                if not v > 0:
                    raise ValueError(f"{key} = {v}")
                vals.append(v)
            return vals[0], vals[1], vals[2], "measured"
        except (OSError, ValueError, TypeError, KeyError) as e:
            print(f"bench: {path} not usable ({e!r}); using the fallback peaks", file=sys.stderr)
    return (*FALLBACK_PEAKS, "fallback")


# ------------------------------------------------------------------ DRAM traffic (ncu)

TRAFFIC_SUMMARY = os.path.join(ROOT, "profiles", "dram_traffic_qwen3_1layer_8192tok.md")
KERNEL_SOURCES = {
    "gemm": ["gemm.cu", "ptx.cuh", "quant_math.cuh", "host_cache.h"],
    "quant": ["quant.cu", "quant_math.cuh", "ptx.cuh", "host_cache.h"],
}


def sources_sha256(kind):
    """Hash of the CUDA sources a kernel family is built from."""
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kind]:
        with open(os.path.join(ROOT, "fp8_blockwise_scaled_e4m3_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def ncu_traffic(kind, algorithmic_bytes_per_launch):
    """DRAM bytes (read + write) per launch of a kernel family in the step, from the committed
    ncu summary of one 8192-token layer (the step's own shapes): that capture's DRAM bytes
    over its algorithmic bytes, times the step's algorithmic bytes per launch. None if there
    is no summary or the family's sources changed since it was captured."""
    try:
        with open(TRAFFIC_SUMMARY) as f:
            text = f.read()
    except OSError:
        return None
    sha = re.search(rf"^{kind}_sources_sha256: ([0-9a-f]{{64}})$", text, re.M)
    val = re.search(rf"^{kind}_dram_over_algorithmic: ([0-9.]+)$", text, re.M)
    if sha is None or val is None or sha.group(1) != sources_sha256(kind):
        return None
    return round(float(val.group(1)) * algorithmic_bytes_per_launch)


# ------------------------------------------------------------------ clocks sampler

class Clocks:
    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        # PURO_CLOCKS_DIR keeps the raw samples; by default they go to a temporary file.
        keep = os.environ.get("PURO_CLOCKS_DIR")
        if keep:
            self.path = os.path.join(keep, f"clocks_gpu{gpu_index}.csv")
        else:
            fd, self.path = tempfile.mkstemp(prefix=f"puro_clocks_gpu{gpu_index}_", suffix=".csv")
            os.close(fd)
        self.temporary = not keep
        self.proc = None
        self.gpu_index = gpu_index

    def _drop(self):
        if self.temporary:
            try:
                os.remove(self.path)
            except OSError:
                pass

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu_index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"], stdout=self.f,
                stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self, t_begin, t_end):
        """Stops sampling; summarises the samples taken between host times t_begin and t_end."""
        import datetime
        if self.proc is None:
            self._drop()
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        sm, mx, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        with open(self.path) as f:
            for line in f:
                c = [x.strip() for x in line.split(",")]
                if len(c) < 9:
                    continue
                try:
                    ts = datetime.datetime.strptime(c[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                    clk, clk_max = float(c[1]), float(c[2])
                except ValueError:
                    continue
                if not (t_begin <= ts <= t_end):
                    continue
                sm.append(clk)
                mx.append(clk_max)
                for name, v in zip(names, c[5:9]):
                    if v.lower() == "active":
                        reasons.add(name)
        self._drop()
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


# ------------------------------------------------------------------ the GPU step

class Step:
    """All buffers of one micro-step and the sequence of library calls over them.

    scales="fp32": the method's scales (amax / 448 as FP32) and the blockwise GEMM;
    scales="pow2": the power-of-two (UE8M0 byte) quantisers and the block-scaled GEMM
    (one wgrad launch per linear: that GEMM has no grouped launch)."""

    def __init__(self, pf, wl, tokens, layers, device, seed, group_wgrad=True, scales="fp32", lm_head=True):
        import torch
        self.pf, self.torch = pf, torch
        if scales not in ("fp32", "pow2"):
            raise ValueError(scales)
        self.scales = scales
        pow2 = scales == "pow2"
        self._qw = pf.puro_fp8_quantize_128x128_pow2 if pow2 else pf.puro_fp8_quantize_128x128
        self._qt = pf.puro_fp8_quantize_1x128_transposed_pow2 if pow2 else pf.puro_fp8_quantize_1x128_transposed
        if pow2:
            self._gemm = lambda a, sa, b, sb, c, lay, st: pf.puro_fp8_mx_gemm(a, sa, b, sb, c, lay, st)
            group_wgrad = False
        else:
            self._gemm = lambda a, sa, b, sb, c, lay, st: pf.puro_fp8_gemm_blockwise(a, sa, b, sb, c, lay, None, st)
        # grouped launches: one per block for its wgrads, one per 64 weights for the weights
        self.group_weights = group_wgrad and not pow2
        T = tokens
        self.tokens = T
        self.linears = []  # (tag, X, W, dY, wq, wqt, ws, xqt, xst) in forward order
        for l in range(layers):
            fwd = wl.layer_forward(seed, T, device, layer=l)
            grads = wl.layer_grads(seed, T, device, layer=l)
            for (name, x, w), (_, dy) in zip(fwd, grads):
                self.linears.append([f"L{l}.{name}", x, w, dy])
        if lm_head:
            h, w_head, dl = wl.lm_head(seed, T, device)
            self.linears.append(["lm_head", h, w_head, dl])
        torch.cuda.synchronize()
        self.scratch = {}
        u8, bf = torch.uint8, torch.bfloat16
        sdt = torch.uint8 if pow2 else torch.float32   # the scales' type
        sb = 1 if pow2 else 4                          # bytes per scale
        for lin in self.linears:
            _, x, w, dy = lin
            n, k = w.shape
            lin += [torch.empty((n, k), dtype=u8, device=device),           # Wq
                    torch.empty((k, n), dtype=u8, device=device),           # WqT
                    torch.empty(((n + 127) // 128, k // 128), dtype=sdt, device=device),  # Ws
                    # X's codes along the tokens, made in the forward, used by wgrad
                    torch.empty((k, T), dtype=u8, device=device),           # XqT
                    torch.empty((T // 128, k), dtype=sdt, device=device)]   # XsT
            if (n, k) not in self.scratch:
                e = lambda *s, dt=u8: torch.empty(s, dtype=dt, device=device)
                self.scratch[(n, k)] = dict(
                    xq=e(T, k), xs=e(k // 128, T, dt=sdt),
                    dyq=e(T, n), dys=e(n // 128, T, dt=sdt),
                    dyqt=e(n, T), dyst=e(T // 128, n, dt=sdt),
                    y=e(T, n, dt=bf), dx=e(T, k, dt=bf), dw=e(n, k, dt=bf))
        self.side = torch.cuda.Stream(device=device)  # weight quantisers and wgrad (overlap mode)
        self.gemm_flops = sum(3 * 2 * T * lin[2].shape[0] * lin[2].shape[1] for lin in self.linears)
        # algorithmic quantiser bytes: BF16 read + code writes + FP32 scale writes
        qb = 0
        for _, x, w, dy, *_ in self.linears:
            n, k = w.shape
            qb += T * k * (2 + 2) + sb * (T * (k // 128) + (T // 128) * k)  # X dual
            qb += n * k * (2 + 2) + sb * (n // 128) * (k // 128)         # W + WqT
            qb += T * n * (2 + 2) + sb * (T * (n // 128) + (T // 128) * n)  # dY dual
        self.quant_bytes = qb
        # algorithmic GEMM bytes: FP8 operands and scales read once, BF16 output written
        gb = 0
        for _, x, w, dy, *_ in self.linears:
            n, k = w.shape
            gb += T * k + n * k + sb * (T * k // 128 + (n // 128) * (k // 128)) + 2 * T * n   # fprop
            gb += T * n + n * k + sb * (T * n // 128 + (n // 128) * (k // 128)) + 2 * T * k   # dgrad
            gb += n * T + k * T + sb * (n + k) * (T // 128) + 2 * n * k                      # wgrad
        self.gemm_bytes = gb
        self.group_wgrad = group_wgrad
        n_wgrad = len({self.layer_of(i) for i in range(len(self.linears))}) if group_wgrad else len(self.linears)
        self.gemm_launches = 2 * len(self.linears) + n_wgrad
        n_wquant = -(-len(self.linears) // 64) if self.group_weights else len(self.linears)
        self.quant_launches = 2 * len(self.linears) + n_wquant
        self.launches_per_step = self.gemm_launches + self.quant_launches

    def run(self, ev=None, stream=None, overlap=False, before_fwd=None, before_bwd=None,
            before_wgrad=None, after_wgrad=None):
        """Enqueue one step on `stream` (default: the current one).

        Order: every weight is quantised first (weights are known before the forward),
        then the forward sweep (quantise X, fprop) and the backward sweep (quantise dY with
        both outputs, quantise X along tokens, dgrad, wgrad). With overlap=True the weight
        quantisers and the wgrads run on a second stream: in a backward pass only dgrad
        feeds the next layer, so wgrad is off the critical path and its kernels fill the
        SMs the other stream's kernels leave idle. Events order every producer before its
        consumers and every reuse of a per-shape scratch buffer after its last reader.

        ev: list to which (kind, event) pairs are appended after each launch (serial mode
        only; an initial event must already be recorded). Hooks, each given the stream its
        next launch goes to: before_fwd(i, st) before linear i's inputs are first read
        (weight quantiser and forward), before_bwd(i, st) before its dY is first read,
        before_wgrad(i, st) before its wgrad writes the shared dW buffer, after_wgrad(i,
        dW, st) right after that wgrad is enqueued."""
        torch, pf = self.torch, self.pf
        if overlap and ev is not None:
            raise ValueError("per-launch events need the serial order")
        main = stream if stream is not None else torch.cuda.current_stream()
        side = self.side if overlap else main
        rec = (lambda kind: ev.append((kind, _record(torch)))) if ev is not None else (lambda kind: None)
        if overlap:
            side.wait_stream(main)  # the previous step is done with every buffer
        w_ready = []
        with torch.cuda.stream(side):
            if self.group_weights and before_fwd is None:
                # every weight is known before the forward: one grouped launch per 64 weights
                pf.puro_fp8_quantize_128x128_grouped([lin[2:3] + lin[4:7] for lin in self.linears], side)
                for _ in range(-(-len(self.linears) // 64)):
                    rec("q")
                w_ready = [side.record_event() if overlap else None] * len(self.linears)
            else:  # per weight, each as soon as its inputs are there (the e2e run's copies)
                for i, (tag, x, w, dy, wq, wqt, ws, xqt, xst) in enumerate(self.linears):
                    if before_fwd is not None:
                        before_fwd(i, side)
                    self._qw(w, wq, wqt, ws, side); rec("q")
                    w_ready.append(side.record_event() if overlap else None)
        for i, (tag, x, w, dy, wq, wqt, ws, xqt, xst) in enumerate(self.linears):
            if before_fwd is not None and overlap:
                before_fwd(i, main)
            s = self.scratch[tuple(w.shape)]
            self._qt(x, xqt, xst, s["xq"], s["xs"], main); rec("q")
            if overlap:
                main.wait_event(w_ready[i])
            self._gemm(s["xq"], s["xs"], wq, ws, s["y"], pf.PURO_FPROP, main); rec("g")
        wgrad_done = {}  # per shape: the last wgrad that read the shape's token-dim operands
        pending = []     # this layer's linears whose dY is quantised and whose wgrad is not issued

        def issue_wgrads():
            # One launch for a layer's wgrads (grouped mode), else one per linear.
            if not pending:
                return
            if overlap:
                side.wait_stream(main)  # every pending dY quantisation is done
            for i in pending:
                if before_wgrad is not None:
                    before_wgrad(i, side)
            with torch.cuda.stream(side):
                probs = []
                for i in pending:
                    _, x, w, dy, wq, wqt, ws, xqt, xst = self.linears[i]
                    s = self.scratch[tuple(w.shape)]
                    probs.append((s["dyqt"], s["dyst"], xqt, xst, s["dw"]))
                if self.group_wgrad and len(probs) > 1:
                    pf.puro_fp8_gemm_blockwise_grouped(probs, pf.PURO_WGRAD, side); rec("g")
                else:
                    for pr in probs:
                        self._gemm(*pr, pf.PURO_WGRAD, side); rec("g")
                if after_wgrad is not None:
                    for i, pr in zip(pending, probs):
                        after_wgrad(i, pr[4], side)
            if overlap:
                done = side.record_event()
                for i in pending:
                    wgrad_done[tuple(self.linears[i][2].shape)] = done
            pending.clear()

        for i in range(len(self.linears) - 1, -1, -1):
            tag, x, w, dy, wq, wqt, ws, xqt, xst = self.linears[i]
            if pending and self.layer_of(pending[-1]) != self.layer_of(i):
                issue_wgrads()
            key = tuple(w.shape)
            s = self.scratch[key]
            if before_bwd is not None:
                before_bwd(i, main)
            if overlap and key in wgrad_done:
                main.wait_event(wgrad_done[key])  # the quantiser below overwrites its dY operands
            self._qt(dy, s["dyqt"], s["dyst"], s["dyq"], s["dys"], main); rec("q")
            self._gemm(s["dyq"], s["dys"], wqt, ws, s["dx"], pf.PURO_DGRAD, main); rec("g")
            pending.append(i)
            if not self.group_wgrad:
                issue_wgrads()
        issue_wgrads()
        if overlap:
            main.wait_stream(side)

    def layer_of(self, i):
        """The block a linear belongs to (its tag's prefix; the LM head is its own)."""
        return self.linears[i][0].split(".")[0]


def _record(torch):
    e = torch.cuda.Event(enable_timing=True)
    e.record()
    return e


def _dist_setup(n_gpus):
    import torch
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return rank, world, local


def _barrier_sync(world):
    import torch
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    if torch.cuda.is_available():
        torch.cuda.synchronize()


def _max_over_ranks(v, world):
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ CPU oracle baseline

def oracle_linear_sample(tokens, seed=0):
    """The oracle on one O-projection linear (2048 -> 2048) over `tokens` tokens: all its
    quantise calls plus fprop, dgrad and wgrad. Returns (GEMM FLOPs, seconds)."""
    from fp8_blockwise_scaled_e4m3_b200 import workloads as wl
    from oracle import gemm as og
    from oracle import quant as oq
    g = wl.generator(seed, 0, "cpu")
    x = wl.bf16_bits(wl.bf16(wl.heavy_tailed((tokens, 2048), 1.0, g, "cpu")))
    w = wl.bf16_bits(wl.bf16(wl.normal((2048, 2048), wl.WEIGHT_STD, g, "cpu")))
    dy = wl.bf16_bits(wl.bf16(wl.heavy_tailed((tokens, 2048), wl.GRAD_STD, g, "cpu")))
    t0 = time.perf_counter()
    xq, xs = oq.quant_1x128(x)
    wq, wqt, ws = oq.quant_128x128(w)
    og.gemm_ref(xq, xs, wq, ws, "fprop")
    dyq, dys = oq.quant_1x128(dy)
    dyt, dyst = oq.quant_1x128_transposed(dy)
    xt, xst = oq.quant_1x128_transposed(x)
    og.gemm_ref(dyq, dys, wqt, ws, "dgrad")
    og.gemm_ref(dyt, dyst, xt, xst, "wgrad")
    dt = time.perf_counter() - t0
    return 3 * 2 * tokens * 2048 * 2048, dt


def _cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(tokens):
    flops, dt = oracle_linear_sample(tokens)
    return {"value": round(flops / dt / 1e12, 6), "unit": "TFLOP/s", "cores": _cpu_threads(),
            "kind": "oracle",
            "sample": f"CPU oracle (NumPy; FP32 quantisers single-threaded, FP64 GEMMs on the BLAS "
                      f"threads) on one O-projection linear 2048->2048 at {tokens} tokens: its quantise "
                      f"calls + fprop/dgrad/wgrad, {flops / 1e9:.1f} GFLOP in {dt:.2f} s"}


def run_reference(args):
    rank, world, _ = _dist_setup(args.gpus)
    if rank != 0:
        return
    tokens = 2048
    for _ in range(args.warmup):
        oracle_linear_sample(tokens)
    flops = dt = 0.0
    for _ in range(args.steps):
        f, t = oracle_linear_sample(tokens)
        flops, dt = flops + f, dt + t
    v = flops / dt / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": round(v, 6), "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(1e3 * dt / args.steps, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "reference_sample": f"O-projection linear at {tokens} tokens per step"},
            "cpu_baseline": {"value": round(v, 6), "unit": "TFLOP/s", "cores": _cpu_threads(), "kind": "oracle",
                             "sample": f"one O-projection linear 2048->2048 at {tokens} tokens per step"},
            "e2e": {"value": round(v, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ main

def run_ours(args):
    import torch
    from fp8_blockwise_scaled_e4m3_b200 import puro_fp8 as pf
    from fp8_blockwise_scaled_e4m3_b200 import workloads as wl

    rank, world, local = _dist_setup(args.gpus)
    device = torch.device("cuda", torch.cuda.current_device())
    hbm_gbs, bf16_tf, bf16_tf_sus, peak_src = _peaks()

    step = Step(pf, wl, args.tokens, args.layers, device, seed=4 + 1000 * rank, group_wgrad=not args.no_group,
                lm_head=not args.no_lm_head)
    # A stream of its own (a CUDA graph cannot be captured on the legacy default stream);
    # every launch, event and collective of this rank runs on it or waits for it.
    stream = torch.cuda.Stream(device=device)
    torch.cuda.set_stream(stream)

    clocks = Clocks(torch.cuda.current_device())
    clocks.start()  # sampling starts before the warm-up; only the timed region is kept
    for _ in range(args.warmup):
        step.run(stream=stream, overlap=True)
    pf.puro_fp8_sync_status()

    # By default the step's 483 launches (both streams, with their events) are captured once
    # into a CUDA graph, and each timed step is one replay of it: the same kernels on the
    # same buffers, without the host issuing each launch.
    graph = None
    if not args.no_graph:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            step.run(stream=stream, overlap=True)
        graph.replay()  # one more warm-up step, through the graph
        torch.cuda.synchronize()
        pf.puro_fp8_sync_status()
    run_step = graph.replay if graph is not None else (lambda: step.run(stream=stream, overlap=True))
    _barrier_sync(world)

    # The timed region: whole steps, CUDA events only at its two ends (an event between
    # launches would stop a kernel from setting up while the previous one finishes).
    t_begin = time.time()
    start = _record(torch)
    for _ in range(args.steps):
        run_step()
    end = _record(torch)
    end.synchronize()
    _barrier_sync(world)
    clk = clocks.stop(t_begin, time.time())
    pf.puro_fp8_sync_status()
    ms_total = start.elapsed_time(end)
    ms_total = _max_over_ranks(ms_total, world)

    # Host enqueue cost: the wall time of issuing one step's launches (argument checks,
    # tensor maps, launches; no synchronisation inside), each step started on an idle GPU
    # so that no launch waits for room in the queue.
    host_ms = []
    for _ in range(3):
        torch.cuda.synchronize()
        h0 = time.perf_counter()
        step.run(stream=stream, overlap=True)
        host_ms.append((time.perf_counter() - h0) * 1e3)
    torch.cuda.synchronize()
    pf.puro_fp8_sync_status()

    # Kernel-level pass after the timed region: an event after every launch gives each
    # kernel's duration for the rooflines.
    kernel_steps = max(1, min(args.steps, 5))
    events = [("start", _record(torch))]
    for _ in range(kernel_steps):
        step.run(ev=events, stream=stream)
    events[-1][1].synchronize()
    pf.puro_fp8_sync_status()
    t_gemm = t_quant = 0.0
    n_gemm = n_quant = 0
    for (_, e0), (kind, e1) in zip(events[:-1], events[1:]):
        dt = e0.elapsed_time(e1)
        if kind == "g":
            t_gemm, n_gemm = t_gemm + dt, n_gemm + 1
        else:
            t_quant, n_quant = t_quant + dt, n_quant + 1

    ms_step = ms_total / args.steps
    value = world * step.gemm_flops / (ms_step * 1e-3) / 1e12
    gemm_tflops = step.gemm_flops * kernel_steps / (t_gemm * 1e-3) / 1e12
    quant_gbs = step.quant_bytes * kernel_steps / (t_quant * 1e-3) / 1e9
    fp8_peak_measured = 2.0 * bf16_tf_sus  # FP8 dense = 2 x BF16 dense (nominal ratio)

    line = {
        "metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "e4m3",
        "data": "synthetic",
        "config": {"workload": workload_name(args), "tokens_per_gpu": args.tokens, "layers": args.layers,
                   "lm_head": not args.no_lm_head, "gemm_tflop_per_step": round(step.gemm_flops / 1e12, 4),
                   "quant_gb_per_step": round(step.quant_bytes / 1e9, 3),
                   "l2": "inputs larger than L2: %.1f GB of distinct BF16 inputs read per step" % (
                       sum(t.numel() * 2 for lin in step.linears for t in lin[1:4]) / 1e9),
                   "parallelism": f"dp{world} (independent micro-batches, no collective)"},
        "frac_of_fp8_peak": round(value / world / FP8_DENSE_PEAK_TFLOPS, 4),
        "roofline": {"bound": "tensor", "kernel": "k_gemm_blockwise (all fprop/dgrad/wgrad launches)",
                     "achieved": round(gemm_tflops, 2), "peak": round(fp8_peak_measured, 1), "unit": "TFLOP/s",
                     "frac": round(gemm_tflops / fp8_peak_measured, 4),
                     "peak_note": f"2 x {peak_src} sustained BF16 ({bf16_tf_sus}); "
                                  f"frac of nominal 4.5 PF = {gemm_tflops / FP8_DENSE_PEAK_TFLOPS:.4f}",
                     "traffic": ncu_traffic("gemm", step.gemm_bytes / step.gemm_launches),
                     "traffic_unit": "DRAM bytes per launch (ncu on one 8192-token layer, scaled to the "
                                     "step's algorithmic bytes per launch)",
                     "algorithmic_bytes_per_launch": round(step.gemm_bytes / step.gemm_launches),
                     "launches_measured": n_gemm, "avg_launch_ms": round(t_gemm / max(n_gemm, 1), 4)},
        "roofline_quant": {"bound": "hbm", "kernel": "k_quant_tiles (dual X and dY, 128x128 weight + WqT launches)",
                           "achieved": round(quant_gbs, 1), "peak": hbm_gbs, "unit": "GB/s",
                           "frac": round(quant_gbs / hbm_gbs, 4),
                           "traffic": ncu_traffic("quant", step.quant_bytes / step.quant_launches),
                           "algorithmic_bytes_per_launch": round(step.quant_bytes / step.quant_launches),
                           "peak_note": f"{peak_src} copy bandwidth; frac of nominal 8 TB/s = "
                                        f"{quant_gbs / 8000:.4f}",
                           "launches_measured": n_quant, "avg_launch_ms": round(t_quant / max(n_quant, 1), 4)},
        "gpu_launches": step.launches_per_step * args.steps,
        "launch": "one CUDA graph replay per step" if graph is not None else "eager launches",
        "host_enqueue_ms_per_step": round(statistics.median(host_ms), 3),
        "clocks": clk,
    }

    # ---------------------------------------------------------------- e2e (host buffers)
    if not args.no_e2e:
        line["e2e"] = run_e2e(step, torch, pf, args, world)

    if rank == 0 and not args.no_cpu_baseline and world == 1:
        line["cpu_baseline"] = cpu_baseline(args.tokens)
    if rank == 0:
        print(json.dumps(line), flush=True)
    del run_step, graph  # released before the process group (it holds no collective)
    torch.cuda.synchronize()
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_e2e(step, torch, pf, args, world):
    """The same step through the public API with host buffers: every step copies the BF16
    inputs (X, W, dY of every linear) from pinned host memory and reads the weight
    gradients back into pinned host memory, inside the timed region. The copies run on
    their own streams in the order the step consumes the tensors (X and W per linear for
    the forward sweep, then dY per linear for the backward sweep), and each linear's
    kernels wait only for their own inputs, so compute overlaps the PCIe transfers."""
    try:
        host_in = []
        for lin in step.linears:
            host_in.append([torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in lin[1:4]])
            for h, t in zip(host_in[-1], lin[1:4]):
                h.copy_(t)
        host_dw = [torch.empty(lin[2].shape, dtype=torch.bfloat16, pin_memory=True) for lin in step.linears]
    except RuntimeError as e:  # pinned host memory exhausted
        return {"unavailable": f"pinned host buffers could not be allocated: {e}"[:200]}
    h2d = sum(t.numel() * t.element_size() for ts in host_in for t in ts)
    d2h = sum(t.numel() * t.element_size() for t in host_dw)

    comp = torch.cuda.current_stream()
    h2d_s, d2h_s = torch.cuda.Stream(), torch.cuda.Stream()
    nlin = len(step.linears)

    def one_step():
        h2d_s.wait_stream(comp)  # the previous step is done with every input buffer
        fwd_ready, bwd_ready = [], [None] * nlin
        with torch.cuda.stream(h2d_s):
            for lin, hs in zip(step.linears, host_in):
                lin[1].copy_(hs[0], non_blocking=True)
                lin[2].copy_(hs[1], non_blocking=True)
                fwd_ready.append(h2d_s.record_event())
            for i in range(nlin - 1, -1, -1):
                step.linears[i][3].copy_(host_in[i][2], non_blocking=True)
                bwd_ready[i] = h2d_s.record_event()
        read_back = {}  # per dW buffer: the read-back that must finish before it is reused

        def before_wgrad(i, st):
            prev = read_back.get(tuple(step.linears[i][2].shape))
            if prev is not None:
                st.wait_event(prev)

        def after_wgrad(i, dw, st):
            d2h_s.wait_event(st.record_event())
            with torch.cuda.stream(d2h_s):
                host_dw[i].copy_(dw, non_blocking=True)
            read_back[tuple(dw.shape)] = d2h_s.record_event()

        step.run(stream=comp, overlap=True, before_fwd=lambda i, st: st.wait_event(fwd_ready[i]),
                 before_bwd=lambda i, st: st.wait_event(bwd_ready[i]), before_wgrad=before_wgrad,
                 after_wgrad=after_wgrad)
        comp.wait_stream(d2h_s)

    one_step()
    comp.synchronize()
    _barrier_sync(world)
    steps = max(1, args.e2e_steps)
    t0 = _record(torch)
    for _ in range(steps):
        one_step()
    t1 = _record(torch)
    t1.synchronize()
    _barrier_sync(world)
    ms = _max_over_ranks(t0.elapsed_time(t1), world) / steps
    return {"value": round(world * step.gemm_flops / (ms * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
            "ms_per_step": round(ms, 3), "steps": steps, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}


def main():
    args = _args()
    if args.impl == "reference":
        run_reference(args)
        return
    if args.config in ("fused", "grouped", "scales", "vendor", "kernels", "nvfp4", "nvfp4-step"):
        import bench_configs
        {"fused": bench_configs.run_fused_comparison, "grouped": bench_configs.run_grouped_comparison,
         "scales": bench_configs.run_scales_comparison, "vendor": bench_configs.run_vendor_reference,
         "kernels": bench_configs.run_kernel_comparison, "nvfp4": bench_configs.run_nvfp4,
         "nvfp4-step": bench_configs.run_nvfp4_step}[args.config](args)
        return
    if args.config in ("1", "2", "3", "4", "all"):
        from bench_configs import run_config
        for c in ((1, 2, 3, 4) if args.config == "all" else (int(args.config),)):
            run_config(c, args)
        if args.config != "all":
            return
    run_ours(args)


if __name__ == "__main__":
    main()
