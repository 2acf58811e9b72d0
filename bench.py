"""Benchmark of the 8-bit quantized linear layer on B200.

Workload (one "step"): the FP8-dynamic decode sweep -- M in {1, 2, 4, 8, 16, 32} tokens
over the four dense-decoder linear shapes (K x N) 4096x6144 (qkv), 4096x4096 (o_proj),
4096x24576 (gate_up), 12288x4096 (down).  For each (M, shape): dynamic per-token fp8
quantization of the bf16 activations, then the scaled FP8 GEMM against per-channel
e4m3 weights -> bf16 out.  48 launches per step, replayed from one CUDA graph.

Metric: achieved HBM TB/s = algorithmic bytes of the step / step time, where a GEMM
moves N*K (weights) + M*K (codes) + 4N + 4M (scales) + 2MN (out) bytes and a quantizer
2MK + MK + 4M.  Weights exist in two copies used alternately (386 MB in total, 3x the
126 MB L2), so no weight matrix is re-read from L2 between its uses.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--detail] [--single KxN --m M]

Under torchrun (N > 1) every rank runs the same workload on its own GPU (the layer
does not shard: replicas only); value = bytes of all ranks / max-over-ranks time.
"""
import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "8-bit GEMM achieved HBM TB/s and % roofline at M=1-32, Qwen3-like shapes"
SHAPES = [(4096, 6144), (4096, 4096), (4096, 24576), (12288, 4096)]   # (K, N)
MS = [1, 2, 4, 8, 16, 32]
WORKLOAD = ("FP8-dynamic decode sweep: per-token e4m3 quant + scaled GEMM, M in {1,2,4,8,16,32} x "
            "(KxN) 4096x6144 qkv, 4096x4096 o_proj, 4096x24576 gate_up, 12288x4096 down")
NCOPY = 2


def gemm_bytes(M, N, K):
    return N * K + M * K + 4 * N + 4 * M + 2 * M * N


def quant_bytes(M, K):
    return 2 * M * K + M * K + 4 * M


def step_bytes(shapes=SHAPES, ms=MS):
    g = sum(gemm_bytes(M, N, K) for M in ms for (K, N) in shapes)
    q = sum(quant_bytes(M, K) for M in ms for (K, N) in shapes)
    return g, q


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            d = json.load(fh)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def gemm_source_hash():
    h = hashlib.sha256()
    for f in ("w8_gemm_kernel.cuh", "w8_gemm.cu", "w8_ptx.cuh", "w8_gemm_decode.cu"):
        with open(os.path.join(ROOT, "bit_quantized_gemm_token_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def traffic_from_profile():
    """DRAM bytes per GEMM launch from the committed ncu summary, or None when the
    summary is missing or was taken on a different GEMM source."""
    p = os.path.join(ROOT, "profiles", "gemm_fp8_decode_sweep_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as fh:
        d = json.load(fh)
    if d.get("gemm_source_sha") != gemm_source_hash():
        return None
    return d.get("dram_bytes_per_launch")


class SmiSampler:
    """nvidia-smi clock / throttle sampling (100 ms) over the whole measurement: the
    fallback when NVML cannot be read."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", self.index, "--query-gpu=" + self.Q,
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None

    def _read(self):
        for ln in self.proc.stdout:
            self.lines.append(ln.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.t.join(timeout=2)
        sm, mx, reasons = [], None, set()
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(ClockSampler.NAMES, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm),
                "source": "nvidia-smi every 100 ms over the measurement"}


class ClockSampler:
    """SM clock and throttle reasons of this GPU during the timed regions.  NVML is read
    (queries only) every millisecond by a thread inside each window, plus one sample
    at each window edge; when NVML cannot be opened, nvidia-smi samples the whole
    measurement instead."""
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
    BITS = {"hw_slowdown": ("nvmlClocksEventReasonHwSlowdown", 0x8),
            "hw_thermal_slowdown": ("nvmlClocksEventReasonHwThermalSlowdown", 0x40),
            "sw_thermal_slowdown": ("nvmlClocksEventReasonSwThermalSlowdown", 0x20),
            "sw_power_cap": ("nvmlClocksEventReasonSwPowerCap", 0x4)}

    def __init__(self, uuid):
        self.sm, self.mx, self.reasons = [], None, set()
        self._nv = self._h = self._smi = self._thr = self._stop = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            self.mx = float(pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM))
            self._get_reasons = (getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None)
                                 or pynvml.nvmlDeviceGetCurrentClocksThrottleReasons)
            self._bits = {n: int(getattr(pynvml, a, b)) for n, (a, b) in self.BITS.items()}
            self._nv = pynvml
        except Exception:
            self._nv = None
            self._smi = SmiSampler(uuid)

    def begin(self):
        if self._smi is not None:
            self._smi.start()

    def _sample(self):
        nv, h = self._nv, self._h
        self.sm.append(float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)))
        r = int(self._get_reasons(h))
        for n, b in self._bits.items():
            if r & b:
                self.reasons.add(n)

    def _poll(self):
        while not self._stop.is_set():
            try:
                self._sample()
            except Exception:
                return
            self._stop.wait(0.001)

    def window_start(self):
        if self._nv is None:
            return
        try:
            self._sample()
        except Exception:
            return
        self._stop = threading.Event()
        self._thr = threading.Thread(target=self._poll, daemon=True)
        self._thr.start()

    def window_stop(self):
        if self._nv is None or self._thr is None:
            return
        self._stop.set()
        self._thr.join(timeout=2)
        self._thr = None
        try:
            self._sample()
        except Exception:
            pass

    def end(self):
        if self._smi is not None:
            return self._smi.stop()
        try:
            self._nv.nvmlShutdown()
        except Exception:
            pass
        if not self.sm:
            return None
        return {"sm_mhz": statistics.median(self.sm), "sm_max_mhz": self.mx, "reasons": sorted(self.reasons),
                "samples": len(self.sm), "source": "NVML every 1 ms inside the timed regions"}


def dist_setup(n_gpus):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(world, v):
    """Largest value over all ranks (the job's time is its slowest rank's)."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world, bytes_per_rank, ms_max):
    """Whole-job TB/s: every rank moves the same bytes (replicas), the job takes the
    slowest rank's time."""
    return world * bytes_per_rank / (ms_max * 1e-3) / 1e12


# --------------------------------------------------------------------------- our arm

class Workload:
    def __init__(self, dev, shapes, ms, seed, ncopy=NCOPY):
        import torch
        from bit_quantized_gemm_token_b200 import w8
        self.w8 = w8
        self.shapes, self.ms = shapes, ms
        g = torch.Generator(device=dev)
        g.manual_seed(seed)
        self.W = {}   # (shape, copy) -> (Wq, sW)
        for (K, N) in shapes:
            for c in range(ncopy):
                wb = (torch.randn(N, K, device=dev, generator=g) * 0.02).to(torch.bfloat16)
                self.W[(K, N, c)] = w8.w8_quant_per_token(wb, w8.W8_Q_FP8)   # per-output-channel
                del wb
        self.X, self.A, self.OUT = {}, {}, {}
        for M in ms:
            for (K, N) in shapes:
                x = torch.randn(M, K, device=dev, generator=g)
                n = M * K
                idx = torch.randint(0, n, (max(1, n // 1000),), device=dev, generator=g)
                x.view(-1)[idx] *= 20.0
                self.X[(M, K, N)] = x.to(torch.bfloat16)
                self.A[(M, K, N)] = (torch.empty((M, K), dtype=torch.float8_e4m3fn, device=dev),
                                     torch.empty((M,), dtype=torch.float32, device=dev))
                self.OUT[(M, K, N)] = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        nb = max(max(w8.w8_gemm_workspace_size(w8.W8_FMT_FP8_DYN, M, N, K, w8.W8_V_PDL),
                     w8.w8_linear_workspace_size(w8.W8_FMT_FP8_DYN, M, N, K, w8.W8_V_PDL))
                 for M in ms for (K, N) in shapes)
        self.ws = w8.Workspace(dev, nb)
        self.path = "pair"
        torch.cuda.synchronize()

    def rotate(self, ncopy):
        """GEMMs of the first (M, shape) against every weight copy in turn."""
        w8 = self.w8
        M, (K, N) = self.ms[0], self.shapes[0]
        q, s = self.A[(M, K, N)]
        w8.w8_quant_per_token(self.X[(M, K, N)], w8.W8_Q_FP8, q=q, scale=s)
        for c in range(ncopy):
            Wq, sW = self.W[(K, N, c)]
            w8.w8_gemm(w8.W8_FMT_FP8_DYN, q, s, Wq, sW, out=self.OUT[(M, K, N)],
                       variant=w8.W8_VARIANT_AUTO | w8.W8_V_PDL, workspace=self.ws)
        return ncopy

    def order(self):
        for mi, M in enumerate(self.ms):
            for si, (K, N) in enumerate(self.shapes):
                yield M, K, N, (mi + si) % NCOPY

    def step(self, quant=True, gemm=True):
        w8 = self.w8
        v = w8.W8_VARIANT_AUTO | w8.W8_V_PDL
        n = 0
        if self.path == "linear" and quant and gemm:
            # quantize + GEMM per layer through w8_linear: the quantizer and the GEMM, or one
            # kernel where the table asks for the fused form
            for M, K, N, c in self.order():
                Wq, sW = self.W[(K, N, c)]
                w8.w8_linear(w8.W8_FMT_FP8_DYN, self.X[(M, K, N)], Wq, sW, out=self.OUT[(M, K, N)], variant=v,
                             workspace=self.ws)
                n += 1 if (w8.w8_linear_resolve(0, M, N, K, v) & w8.W8_V_FUSED) else 2
            return n
        for M, K, N, c in self.order():
            q, s = self.A[(M, K, N)]
            if quant:
                w8.w8_quant_per_token(self.X[(M, K, N)], w8.W8_Q_FP8, q=q, scale=s)
                n += 1
            if gemm:
                Wq, sW = self.W[(K, N, c)]
                w8.w8_gemm(w8.W8_FMT_FP8_DYN, q, s, Wq, sW, out=self.OUT[(M, K, N)], variant=v, workspace=self.ws)
                n += 1
        return n


def time_graph(fn, steps, warmup, world, clock=None):
    """Capture fn() into a CUDA graph, replay `warmup` times, then time `steps` replays
    with CUDA events on the capturing stream (the clock sampler, if any, samples that
    window).  Returns (ms per step, launches per step)."""
    import torch
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()                      # eager warm-up (module load, smem attributes)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        launches = fn()
    for _ in range(warmup):
        g.replay()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    if clock is not None:
        clock.window_start()
    with torch.cuda.stream(s):
        e0.record(s)
        for _ in range(steps):
            g.replay()
        e1.record(s)
    torch.cuda.synchronize()
    if clock is not None:
        clock.window_stop()
    ms = e0.elapsed_time(e1) / steps
    barrier(world)
    del g
    return ms, launches


BLOCK_SHAPES = [(5120, 10240), (5120, 51200), (25600, 5120), (4096, 6144)]


def short_variant(v):
    from bit_quantized_gemm_token_b200 import w8
    d = w8.describe(v)
    if d["decode"]:
        return "decode bn%d c%d st%d" % (d["bn"], d["c"], d["stages"])
    form = "pair" if d["pair"] else "swap" if d["swap_ab"] else "std"
    part = "stream" if d["stream"] else ("cluster%d" % d["split_k"]) if d["cluster"] else ("split%d" % d["split_k"])
    return "%s bn%d %s" % (form, d["bn"], part)


def time_decode_table(dev, peak, reps=10):
    """Every (format, shape, M) of the decode workloads timed alone: the GEMM (AUTO +
    programmatic dependent launch) replayed from a CUDA graph against enough weight copies
    to exceed 3x the L2, so each launch streams its weights from HBM.  Per entry: K, N, M,
    microseconds, TB/s of algorithmic bytes and the fraction of the measured copy peak,
    and the variant AUTO resolved to; per format the weight-byte-weighted aggregate
    (total bytes / total time)."""
    import torch
    from bit_quantized_gemm_token_b200 import w8
    g = torch.Generator(device=dev)
    g.manual_seed(777)
    out = {}
    for name, fmt, shapes in (("fp8_dynamic", w8.W8_FMT_FP8_DYN, SHAPES), ("w8a8_int8", w8.W8_FMT_INT8, SHAPES),
                              ("block_fp8", w8.W8_FMT_BLOCK_FP8, BLOCK_SHAPES)):
        block = fmt >= w8.W8_FMT_BLOCK_FP8
        rows, tot_b, tot_us = [], 0, 0.0
        for (K, N) in shapes:
            ncopy = max(2, -(-400_000_000 // (N * K)))
            W = []
            for _ in range(ncopy):
                wb = (torch.randn(N, K, device=dev, generator=g) * 0.02).to(torch.bfloat16)
                W.append(w8.w8_quant_weight_block(wb) if block else
                         w8.w8_quant_per_token(wb, w8.W8_Q_INT8 if fmt == w8.W8_FMT_INT8 else w8.W8_Q_FP8))
                del wb
            ws = w8.Workspace(dev)
            for M in MS:
                x = torch.randn(M, K, device=dev, generator=g).to(torch.bfloat16)
                if block:
                    A, sA = w8.w8_quant_per_token(x, w8.W8_Q_FP8, group=128)
                else:
                    A, sA = w8.w8_quant_per_token(x, w8.W8_Q_INT8 if fmt == w8.W8_FMT_INT8 else w8.W8_Q_FP8)
                o = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
                v = w8.W8_VARIANT_AUTO | w8.W8_V_PDL

                def rot():
                    for Wq, sW in W:
                        w8.w8_gemm(fmt, A, sA, Wq, sW, out=o, variant=v, workspace=ws)
                    return len(W)
                ms, n = time_graph(rot, reps, 3, 1)
                us = ms * 1e3 / n
                if block:
                    b = N * K + 4 * ((N + 127) // 128) * (K // 128) + M * K + 4 * M * (K // 128) + 2 * M * N
                else:
                    b = gemm_bytes(M, N, K)
                tot_b += b
                tot_us += us
                tbs = b / us / 1e6
                rows.append([K, N, M, round(us, 2), round(tbs, 3), round(tbs * 1e3 / peak, 4),
                             short_variant(w8.w8_gemm_resolve_variant(fmt, M, N, K))])
            del W, ws
            torch.cuda.empty_cache()
        agg = tot_b / tot_us / 1e6
        out[name] = {"rows": rows, "weighted_TB/s": round(agg, 3), "weighted_frac": round(agg * 1e3 / peak, 4)}
    out["columns"] = ["K", "N", "M", "us", "TB/s", "frac of measured copy peak", "variant"]
    return out


def time_extras(dev, peak):
    """Device time of the other hot-path kernels on their own (CUDA graph of a few launches
    over inputs rotated past L2): the query/key rms_norm + rotary embedding at prefill size,
    and the grouped (mixture-of-experts) GEMM at a decode routing.  HBM roofline fractions
    against the same measured copy peak."""
    import torch
    from bit_quantized_gemm_token_b200 import w8
    g = torch.Generator(device=dev)
    g.manual_seed(4242)
    res = {}
    # qk norm + rope: 4096 tokens, 32 query / 8 key-value heads of 128 (in place)
    T, Hq, Hkv, D = 4096, 32, 8, 128
    bufs = [(torch.randn(T, (Hq + 2 * Hkv) * D, device=dev, generator=g)).to(torch.bfloat16) for _ in range(3)]
    qw = (torch.rand(D, device=dev, generator=g) + 0.5).to(torch.bfloat16)
    kw = (torch.rand(D, device=dev, generator=g) + 0.5).to(torch.bfloat16)
    pos = torch.randint(0, 8192, (T,), device=dev, generator=g)
    ang = torch.rand(8192, D // 2, device=dev, generator=g) * 6.283
    table = torch.cat([ang.cos(), ang.sin()], dim=1).float()

    def qk():
        for b in bufs:
            w8.w8_qk_norm_rope(b, Hq, Hkv, D, qw, kw, table, pos, out=b, stream=torch.cuda.current_stream())
        return len(bufs)
    ms, n = time_graph(qk, 5, 3, 1)
    us = ms * 1e3 / n
    byts = T * (Hq + Hkv) * D * 2 * 2 + T * D * 4
    res["qk_norm_rope"] = {"shape": "T=%d Hq=%d Hkv=%d D=%d, in place" % (T, Hq, Hkv, D), "us": round(us, 2),
                           "GB/s": round(byts / (us * 1e-6) / 1e9, 1),
                           "frac": round(byts / (us * 1e-6) / 1e9 / peak, 4), "bytes": byts}
    # grouped GEMM: 128 experts of 1536 x 2048 (FP8), 4 tokens routed to 8 experts each
    E, N, K, M, top = 128, 1536, 2048, 4, 8
    sets = []
    for _ in range(2):
        wb = (torch.randn(E * N, K, device=dev, generator=g) * 0.02).to(torch.bfloat16)
        Wq, sW = w8.w8_quant_per_token(wb, w8.W8_Q_FP8)
        sets.append((Wq.view(E, N, K), sW.view(E, N)))
        del wb
    choice = torch.stack([torch.randperm(E, device=dev, generator=g)[:top] for _ in range(M)]).flatten()
    counts = torch.bincount(choice, minlength=E)
    off = torch.zeros(E + 1, dtype=torch.int32, device=dev)
    off[1:] = torch.cumsum(counts, 0).to(torch.int32)
    rows = M * top
    A = (torch.randn(rows, K, device=dev, generator=g)).to(torch.bfloat16)
    Aq, sA = w8.w8_quant_per_token(A, w8.W8_Q_FP8)
    out = torch.empty(rows, N, dtype=torch.bfloat16, device=dev)
    ws = w8.Workspace(dev)
    active = int((counts > 0).sum().item())

    def grouped():
        for Wq, sW in sets:
            w8.w8_grouped_gemm(w8.W8_FMT_FP8_DYN, Aq, sA, Wq, sW, off, max_tokens_per_expert=M, out=out,
                               variant=w8.W8_VARIANT_AUTO | w8.W8_V_PDL, workspace=ws)
        return len(sets)
    ms, n = time_graph(grouped, 5, 3, 1)
    us = ms * 1e3 / n
    byts = active * N * K + rows * K + 4 * active * N + 4 * rows + 2 * rows * N
    res["grouped_gemm"] = {"shape": "E=%d N=%d K=%d, %d tokens x top-%d -> %d active experts" % (E, N, K, M, top, active),
                           "us": round(us, 2), "GB/s": round(byts / (us * 1e-6) / 1e9, 1),
                           "frac": round(byts / (us * 1e-6) / 1e9 / peak, 4), "bytes": byts}
    del sets
    torch.cuda.empty_cache()
    # prefill GEMM (tensor-bound): FP8-dynamic, M = 4096 tokens on the gate_up shape
    M, K, N = 4096, 4096, 24576
    Aq, sA = w8.w8_quant_per_token(torch.randn(M, K, device=dev, generator=g).to(torch.bfloat16), w8.W8_Q_FP8)
    Wq, sW = w8.w8_quant_per_token((torch.randn(N, K, device=dev, generator=g) * 0.02).to(torch.bfloat16), w8.W8_Q_FP8)
    out = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    flop = 2.0 * M * N * K
    fp8_peak = 2.0 * peak_tflops()          # dense fp8 = 2 x the measured dense bf16 figure
    best = None
    tried = {}
    for name, v in [("auto", w8.W8_VARIANT_AUTO), ("standard 128x256", w8.variant(False, 1, 256)),
                    ("standard 128x128", w8.variant(False, 1, 128)), ("balanced 128x256", w8.variant(False, 1, 256, stream=True)),
                    ("CTA pairs 256x256", w8.variant(False, 1, 256, pair=True)),
                    ("CTA pairs 256x256, 6 stages", w8.variant(False, 1, 256, pair=True, stages=6))]:
        def pre():
            for _ in range(3):
                w8.w8_gemm(w8.W8_FMT_FP8_DYN, Aq, sA, Wq, sW, out=out, variant=v | w8.W8_V_PDL, workspace=ws)
            return 3
        ms, n = time_graph(pre, 3, 2, 1)
        tf = flop / (ms * 1e-3 / n) / 1e12
        tried[name] = round(tf, 1)
        if best is None or tf > best[1]:
            best = (name, tf, ms * 1e3 / n)
    res["prefill_gemm"] = {"shape": "FP8-dynamic M=%d K=%d N=%d" % (M, K, N), "variant": best[0], "us": round(best[2], 1),
                           "TFLOP/s": round(best[1], 1), "peak_TFLOP/s": round(fp8_peak, 1),
                           "frac": round(best[1] / fp8_peak, 4),
                           "peak_source": "2 x measured dense bf16 (burst)", "variants_TFLOP/s": tried}
    # the same shape in W8A8-INT8 (int8 tensor cores, int32 accumulation), built-in variant
    xa = torch.randn(M, K, device=dev, generator=g).to(torch.bfloat16)
    xw = (torch.randn(N, K, device=dev, generator=g) * 0.02).to(torch.bfloat16)
    Aq, sA = w8.w8_quant_per_token(xa, w8.W8_Q_INT8)
    Wq, sW = w8.w8_quant_per_token(xw, w8.W8_Q_INT8)
    del xa, xw

    def pre_i8():
        for _ in range(3):
            w8.w8_gemm(w8.W8_FMT_INT8, Aq, sA, Wq, sW, out=out, variant=w8.W8_VARIANT_AUTO | w8.W8_V_PDL, workspace=ws)
        return 3
    ms, n = time_graph(pre_i8, 3, 2, 1)
    tf = flop / (ms * 1e-3 / n) / 1e12
    res["prefill_gemm_int8"] = {"shape": "W8A8-INT8 M=%d K=%d N=%d" % (M, K, N), "us": round(ms * 1e3 / n, 1),
                                "TOP/s": round(tf, 1), "peak_TOP/s": round(fp8_peak, 1), "frac": round(tf / fp8_peak, 4),
                                "peak_source": "2 x measured dense bf16 (burst)"}
    del Aq, Wq, out
    torch.cuda.empty_cache()
    # the other formats' decode chains (quantizer + GEMM per layer), like the step above
    res["int8_decode"] = format_chain(dev, g, w8, w8.W8_FMT_INT8, SHAPES, [1, 8, 32], peak)
    res["block_fp8_decode"] = format_chain(dev, g, w8, w8.W8_FMT_BLOCK_FP8,
                                           [(5120, 10240), (5120, 51200), (25600, 5120), (4096, 6144)], [1, 8, 32], peak)
    res["mlp_chain"] = mlp_chain(dev, g, w8, peak, fp8_peak)
    res["mlp_chain_block_fp8"] = mlp_chain(dev, g, w8, peak, fp8_peak, fmt=w8.W8_FMT_BLOCK_FP8)
    return res


def mlp_chain(dev, g, w8, peak, fp8_peak, fmt=0):
    """The MLP block hidden 4096 / intermediate 12288: rms_norm + quant, gate_up GEMM,
    silu_and_mul + quant, down GEMM (AUTO + PDL, one CUDA graph per token count, two
    weight copies in rotation), in FP8-dynamic (per-token scales, per-channel weights) or
    Block-FP8 (fmt 2: 1 x 128 activation groups, 128 x 128 weight blocks).  Decode token
    counts in TB/s of algorithmic bytes, prefill ones in TFLOP/s of the two GEMMs."""
    import torch
    H, I = 4096, 12288
    block = fmt >= 2
    gamma = (torch.rand(H, device=dev, generator=g) + 0.5).to(torch.bfloat16)
    wq = (lambda wb: w8.w8_quant_weight_block(wb)) if block else (lambda wb: w8.w8_quant_per_token(wb))
    Wgu, Wd = [], []
    for _ in range(2):
        Wgu.append(wq((torch.randn(2 * I, H, device=dev, generator=g) * 0.02).to(torch.bfloat16)))
        Wd.append(wq((torch.randn(H, I, device=dev, generator=g) * 0.02).to(torch.bfloat16)))
    ws = w8.Workspace(dev)
    v = w8.W8_VARIANT_AUTO | w8.W8_V_PDL
    out = {}
    for M in ((1, 8, 32, 256, 1024) if block else (1, 8, 32, 256, 1024, 4096)):
        x = torch.randn(M, H, device=dev, generator=g).to(torch.bfloat16)
        q1 = torch.empty(M, H, dtype=torch.float8_e4m3fn, device=dev)
        s1 = torch.empty(M, H // 128, device=dev) if block else torch.empty(M, device=dev)
        gu = torch.empty(M, 2 * I, dtype=torch.bfloat16, device=dev)
        q2 = torch.empty(M, I, dtype=torch.float8_e4m3fn, device=dev)
        s2 = torch.empty(M, I // 128, device=dev) if block else torch.empty(M, device=dev)
        y = torch.empty(M, H, dtype=torch.bfloat16, device=dev)
        reps = 4 if M <= 32 else 2

        def chain():
            for r in range(reps):
                if block:
                    w8.w8_rmsnorm_quant_group(x, gamma, 1e-6, q=q1, scale=s1)
                else:
                    w8.w8_rmsnorm_quant(x, gamma, 1e-6, q=q1, scale=s1)
                w8.w8_gemm(fmt, q1, s1, Wgu[r % 2][0], Wgu[r % 2][1], out=gu, variant=v, workspace=ws)
                if block:
                    w8.w8_silu_mul_quant_group(gu, q=q2, scale=s2)
                else:
                    w8.w8_silu_mul_quant(gu, q=q2, scale=s2)
                w8.w8_gemm(fmt, q2, s2, Wd[r % 2][0], Wd[r % 2][1], out=y, variant=v, workspace=ws)
            return 4 * reps
        ms, _ = time_graph(chain, 5, 3, 1)
        us = ms * 1e3 / reps
        if M <= 32:
            if block:   # group scales of the activations, 128 x 128 block scales of the weights
                byts = (2 * M * H + 2 * H + M * H + 4 * M * H // 128) \
                    + (2 * I * H + 4 * (2 * I // 128) * (H // 128) + M * H + 4 * M * H // 128 + 2 * M * 2 * I) \
                    + (2 * M * 2 * I + M * I + 4 * M * I // 128) \
                    + (H * I + 4 * (H // 128) * (I // 128) + M * I + 4 * M * I // 128 + 2 * M * H)
            else:
                byts = (2 * M * H + 2 * H + M * H + 4 * M) + gemm_bytes(M, 2 * I, H) \
                    + (2 * M * 2 * I + M * I + 4 * M) + gemm_bytes(M, H, I)
            gbs = byts / (us * 1e-6) / 1e9
            out["M=%d" % M] = {"us": round(us, 2), "GB/s": round(gbs, 1), "frac": round(gbs / peak, 4)}
        else:
            tf = 2.0 * M * (H * 2 * I + I * H) / (us * 1e-6) / 1e12
            out["M=%d" % M] = {"us": round(us, 1), "TFLOP/s": round(tf, 1), "frac": round(tf / fp8_peak, 4)}
        del x, q1, s1, gu, q2, s2, y
    del Wgu, Wd
    torch.cuda.empty_cache()
    out["shape"] = "hidden 4096, intermediate 12288, %s; decode frac of the copy peak, prefill of 2 x dense bf16" % (
        "Block-FP8 (1x128 activation groups, 128x128 weight blocks)" if block else "FP8-dynamic")
    return out


def format_chain(dev, g, w8, fmt, shapes, ms, peak):
    """TB/s of a graph of (activation quantizer, GEMM) pairs over the shapes and token
    counts in format fmt (W8A8-INT8 per token, or Block-FP8 with 1 x 128 activation
    groups and 128 x 128 weight blocks), two weight copies per shape in rotation."""
    import torch
    block = fmt >= w8.W8_FMT_BLOCK_FP8
    W = {}
    for (K, N) in shapes:
        for c in range(2):
            wb = (torch.randn(N, K, device=dev, generator=g) * 0.02).to(torch.bfloat16)
            W[(K, N, c)] = w8.w8_quant_weight_block(wb) if block else w8.w8_quant_per_token(wb, w8.W8_Q_INT8)
            del wb
    X = {(M, K): (torch.randn(M, K, device=dev, generator=g)).to(torch.bfloat16) for M in ms for (K, N) in shapes}
    A = {}
    for (M, K), x in X.items():
        A[(M, K)] = (w8.w8_quant_per_token(x, w8.W8_Q_FP8, group=128) if block else w8.w8_quant_per_token(x, w8.W8_Q_INT8))
    O = {(M, N): torch.empty(M, N, dtype=torch.bfloat16, device=dev) for M in ms for (K, N) in shapes}
    ws = w8.Workspace(dev)
    v = w8.W8_VARIANT_AUTO | w8.W8_V_PDL
    byts = 0
    for M in ms:
        for (K, N) in shapes:
            if block:   # 128 x 128 weight-block scales, 1 x 128 activation-group scales
                kb = K // 128
                byts += (N * K + 4 * ((N + 127) // 128) * kb + M * K + 4 * M * kb + 2 * M * N
                         + 2 * M * K + M * K + 4 * M * kb)
            else:
                byts += gemm_bytes(M, N, K) + quant_bytes(M, K)

    def chain():
        n = 0
        for mi, M in enumerate(ms):
            for si, (K, N) in enumerate(shapes):
                q, sc = A[(M, K)]
                if block:
                    w8.w8_quant_per_token(X[(M, K)], w8.W8_Q_FP8, group=128, q=q, scale=sc)
                else:
                    w8.w8_quant_per_token(X[(M, K)], w8.W8_Q_INT8, q=q, scale=sc)
                Wq, sW = W[(K, N, (mi + si) % 2)]
                w8.w8_gemm(fmt, q, sc, Wq, sW, out=O[(M, N)], variant=v, workspace=ws)
                n += 2
        return n
    ms_step, _ = time_graph(chain, 5, 3, 1)
    tbs = byts / (ms_step * 1e-3) / 1e12
    out = {"shapes_KxN": ["%dx%d" % s for s in shapes], "M": ms, "us_per_step": round(ms_step * 1e3, 1),
           "TB/s": round(tbs, 3), "frac": round(tbs * 1e3 / peak, 4)}
    del W, X, A, O
    torch.cuda.empty_cache()
    return out


def peak_tflops():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            return float(json.load(fh)["bf16_tflops"])
    return 1590.0


def time_e2e(wl, steps, warmup, world):
    """Same step through the public API with host buffers: every step copies each layer's
    activations from pinned host memory to the device, runs its quantize + GEMM calls, and
    copies its output back to pinned host memory.  The copies run on two side streams,
    pipelined with the layers (a layer starts once its input has landed; its output is
    copied back while the next layers run), and the whole step is captured once into a
    CUDA graph and replayed, as a decode loop replays its captured step.  CUDA events on
    the stream around the replays."""
    import torch
    w8 = wl.w8
    keys = [(M, K, N) for M, K, N, c in wl.order()]
    dev = wl.X[keys[0]].device
    hx = {k: wl.X[k].cpu().pin_memory() for k in keys}
    dx = {k: torch.empty_like(wl.X[k]) for k in keys}
    ho = {k: torch.empty(wl.OUT[k].shape, dtype=torch.bfloat16).pin_memory() for k in keys}
    h2d = sum(t.numel() * t.element_size() for t in hx.values())
    d2h = sum(t.numel() * t.element_size() for t in ho.values())
    v = w8.W8_VARIANT_AUTO | w8.W8_V_PDL
    s = torch.cuda.Stream()
    s_in = torch.cuda.Stream()
    s_out = torch.cuda.Stream()

    def one():
        cur = torch.cuda.current_stream()
        s_in.wait_stream(cur)
        s_out.wait_stream(cur)
        landed = {}
        with torch.cuda.stream(s_in):
            for k in keys:
                dx[k].copy_(hx[k], non_blocking=True)
                landed[k] = torch.cuda.Event()
                landed[k].record(s_in)
        for M, K, N, c in wl.order():
            key = (M, K, N)
            cur.wait_event(landed[key])
            q, sc = w8.w8_quant_per_token(dx[key], w8.W8_Q_FP8, q=wl.A[key][0], scale=wl.A[key][1])
            Wq, sW = wl.W[(K, N, c)]
            w8.w8_gemm(w8.W8_FMT_FP8_DYN, q, sc, Wq, sW, out=wl.OUT[key], variant=v, workspace=wl.ws)
            done = torch.cuda.Event()
            done.record(cur)
            s_out.wait_event(done)
            with torch.cuda.stream(s_out):
                ho[key].copy_(wl.OUT[key], non_blocking=True)
        cur.wait_stream(s_in)
        cur.wait_stream(s_out)

    with torch.cuda.stream(s):
        one()                     # eager warm-up
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        one()
    for _ in range(warmup):
        g.replay()
    torch.cuda.synchronize()
    barrier(world)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(s):
        e0.record(s)
        for _ in range(steps):
            g.replay()
        e1.record(s)
    torch.cuda.synchronize()
    del g
    return e0.elapsed_time(e1) / steps, h2d, d2h


class OracleSample:
    """The CPU oracle as it stands (single-threaded C, fp64 GEMM) on a bounded sample of
    the same workload: for every (M, shape) pair, per-token quantization of the full
    activations and the first `cols` output columns of the GEMM.  Throughput is given in
    the metric's unit: algorithmic bytes of the sampled work (weight rows of the
    sampled columns, codes, scales, outputs, quantizer traffic) / time."""

    def __init__(self, shapes, ms):
        import oracle as orc
        from bit_quantized_gemm_token_b200 import synth
        self.orc = orc
        self.shapes, self.ms = shapes, ms
        self.data = {}
        for (K, N) in shapes:
            w = synth.weights(1024, K, seed=synth.SEED_BASE + 2 + N)
            wq, ws = orc.quant_rows(0, synth.bf16_bits(w))
            for M in ms:
                x = synth.activations(M, K, seed=synth.SEED_BASE + 2 + M * 100 + K)
                self.data[(M, K, N)] = (synth.bf16_bits(x), wq, ws)
        self.cols = 64

    def run(self):
        nbytes = 0
        t0 = time.perf_counter()
        for M in self.ms:
            for (K, N) in self.shapes:
                xb, wq, ws = self.data[(M, K, N)]
                aq, sa = self.orc.quant_rows(0, xb)
                self.orc.gemm(0, aq, sa, wq[:self.cols], ws[:self.cols])
                nbytes += quant_bytes(M, K) + gemm_bytes(M, self.cols, K)
        return nbytes, time.perf_counter() - t0

    def size_for(self, seconds):
        """Grow the column sample until one run takes about `seconds`."""
        nb, dt = self.run()
        if dt < seconds:
            self.cols = int(min(1024, max(self.cols, self.cols * seconds / max(dt, 1e-3))))
            nb, dt = self.run()
        return nb, dt

    def describe(self, dt):
        return ("all %d (M, shape) pairs of the workload: per-token quant of the full activations + the first "
                "%d output columns of each GEMM (fp64 triple loop); %.1f s per sample"
                % (len(self.ms) * len(self.shapes), self.cols, dt))


def cpu_baseline(shapes, ms, target_s=10.0):
    smp = OracleSample(shapes, ms)
    nb, dt = smp.size_for(target_s)
    return {"value": nb / dt / 1e12, "unit": "TB/s", "cores": 1, "kind": "oracle", "sample": smp.describe(dt)}


def run_ours(args):
    import torch
    from bit_quantized_gemm_token_b200 import w8
    w8.lib()   # raises if the CUDA library is not built: there is no fallback
    world, rank, local = dist_setup(args.gpus)
    dev = torch.device("cuda", torch.cuda.current_device())
    shapes, ms = SHAPES, MS
    workload = WORKLOAD
    if args.single:
        K, N = (int(v) for v in args.single.lower().split("x"))
        shapes, ms = [(K, N)], [args.m]
        workload = "single FP8-dynamic quant + GEMM, M=%d, KxN=%dx%d" % (args.m, K, N)
    wl = Workload(dev, shapes, ms, seed=1234 + 1 + rank)
    wl.path = args.path
    gb, qb = step_bytes(shapes, ms)

    try:
        gpu_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        gpu_id = str(torch.cuda.current_device())
    clk = ClockSampler(gpu_id) if rank == 0 and not args.no_clocks else None
    if clk:
        clk.begin()
    ms_step, launches = time_graph(lambda: wl.step(True, True), args.steps, args.warmup, world, clk)
    ms_gemm, n_gemm = time_graph(lambda: wl.step(False, True), args.steps, args.warmup, world, clk)
    clocks = clk.end() if clk else None
    ms_step = max_over_ranks(world, ms_step)
    ms_gemm = max_over_ranks(world, ms_gemm)

    e2e = None
    if not args.no_e2e:
        ms_e2e, h2d, d2h = time_e2e(wl, max(1, args.steps // 2), max(1, args.warmup // 2), world)
        ms_e2e = max_over_ranks(world, ms_e2e)
        e2e = {"value": round(job_throughput(world, gb + qb, ms_e2e), 4), "unit": "TB/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(ms_e2e, 4),
               "path": "per layer: pinned-host copy in, w8_quant_per_token + w8_gemm (AUTO + PDL), copy out; the "
                       "copies pipelined with the layers on side streams; the step captured in a CUDA graph"}

    detail = None
    if args.detail and rank == 0:
        detail = []
        for (K, N) in shapes:
            for M in ms:
                ncopy = max(2, -(-400_000_000 // (N * K)))     # > 3x L2 of weights in rotation
                sub = Workload(dev, [(K, N)], [M], seed=99, ncopy=ncopy)
                t, nl = time_graph(lambda: sub.rotate(ncopy), 5, 3, 1)
                t /= nl
                b = gemm_bytes(M, N, K)
                detail.append({"K": K, "N": N, "M": M, "us": round(t * 1e3, 2), "TB/s": round(b / (t * 1e-3) / 1e12, 3),
                               "variant": w8.describe(w8.w8_gemm_resolve_variant(0, M, N, K))})
                del sub

    peak, peak_kind = load_peaks()
    achieved = gb / (ms_gemm * 1e-3) / 1e9    # GB/s, GEMM kernels alone
    n_gemm_per_step = len(shapes) * len(ms)
    # the committed capture is of the decode sweep's GEMM launches: no figure for other workloads
    traffic = traffic_from_profile() if (not args.single and args.path == "pair") else None
    value = job_throughput(world, gb + qb, ms_step)
    out = {
        "metric": METRIC, "value": round(value, 4), "unit": "TB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "e4m3", "data": "synthetic",
        "config": {"workload": workload, "parallelism": "replicas" if world > 1 else "single GPU",
                   "l2": "inputs larger than L2: %d weight copies per shape used alternately (%.0f MB of weights)"
                         % (NCOPY, sum(N * K for (K, N) in shapes) * NCOPY / 1e6),
                   "launch": "CUDA graph of the step; GEMM variant AUTO + programmatic dependent launch",
                   "bytes_per_step": gb + qb},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "peak_source": peak_kind,
                     "traffic": (round(traffic) if traffic is not None else None),
                     "algorithmic_bytes_per_launch": round(gb / n_gemm_per_step),
                     "kernel": "gemm_decode_kernel (w8_gemm FP8-dynamic, decode form)", "ms_gemm_per_step": round(ms_gemm, 4),
                     "frac_of_8TBs": round(achieved / 8000.0, 4)},
        "gpu_launches": launches * args.steps,
    }
    if clocks:
        out["clocks"] = clocks
    if e2e:
        out["e2e"] = e2e
    if detail:
        out["detail"] = detail
    # single-GPU timings of the other kernels: at N = 1 only (with more ranks the others
    # would sit idle, holding their GPUs, while rank 0 times them)
    if rank == 0 and world == 1 and not args.no_extras:
        out["other_kernels"] = time_extras(dev, peak)
        out["kernels"] = time_kernels(dev, peak, peak_tflops())
    if rank == 0 and world == 1 and not args.no_table:
        out["decode_table"] = time_decode_table(dev, peak)
    if rank == 0 and world == 1 and not args.no_cpu:
        out["cpu_baseline"] = cpu_baseline(shapes, ms, target_s=args.cpu_seconds)
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# --------------------------------------------------------------------------- reference arm

def run_reference(args):
    """The reference arm is the CPU oracle as it stands (the pages ship no runnable
    code): each step is one bounded sample of the same workload on the host cores, in
    the same metric and unit.  Under torchrun only rank 0 runs and prints."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    smp = OracleSample(SHAPES, MS)
    smp.size_for(max(0.5, args.ref_seconds))       # sizing run (counts as warm-up)
    for _ in range(max(0, args.warmup - 1)):
        smp.run()
    tot_b, tot_t = 0, 0.0
    for _ in range(args.steps):
        nb, dt = smp.run()
        tot_b += nb
        tot_t += dt
    val = tot_b / tot_t / 1e12
    out = {"impl": "reference", "metric": METRIC, "value": round(val, 9), "unit": "TB/s", "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(tot_t / args.steps * 1e3, 3),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": {"workload": WORKLOAD, "parallelism": "one host thread"},
           "cpu_baseline": {"kind": "oracle", "cores": 1, "sample": smp.describe(tot_t / args.steps),
                            "value": round(val, 9), "unit": "TB/s"},
           "e2e": {"value": round(val, 9), "unit": "TB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


KERNEL_CASES = ("quant_rows", "quant_rows_int8", "group128", "rmsnorm_quant", "silu_mul_quant", "qk_norm_rope",
                "gemm_fp8", "gemm_int8", "gemm_block", "grouped", "pair_prefill")


def kernel_case(case, dev, g):
    """One hot-path kernel on a profiling-sized case: (launch function, algorithmic bytes
    per launch, FLOPs per launch or 0).  The quantizers and producers at 16384 (silu: 4096)
    rows, query/key norm + rotary embedding at 16384 tokens, the decode GEMMs at M = 8 on
    4096 x 24576 (Block-FP8: 5120 x 51200), the grouped GEMM at a decode routing, the
    prefill GEMM at M = 4096.  Bytes count each input once and each output once."""
    import torch
    from bit_quantized_gemm_token_b200 import w8
    def rnd(*shape, scale=1.0):
        return (torch.randn(*shape, device=dev, generator=g) * scale).to(torch.bfloat16)
    flops = 0
    if case in ("quant_rows", "quant_rows_int8", "group128"):
        M, K = 16384, 4096
        x = rnd(M, K)
        grp = 128 if case == "group128" else 0
        qf = w8.W8_Q_INT8 if case == "quant_rows_int8" else w8.W8_Q_FP8
        q = torch.empty(M, K, dtype=torch.int8 if qf == w8.W8_Q_INT8 else torch.float8_e4m3fn, device=dev)
        s = torch.empty(M, K // 128, device=dev) if grp else torch.empty(M, device=dev)
        f = lambda: w8.w8_quant_per_token(x, qf, group=grp, q=q, scale=s)
        byts = M * K * 3 + s.numel() * 4
    elif case == "rmsnorm_quant":
        M, H = 16384, 4096
        x = rnd(M, H); gm = (torch.rand(H, device=dev, generator=g) + 0.5).to(torch.bfloat16)
        q = torch.empty(M, H, dtype=torch.float8_e4m3fn, device=dev); s = torch.empty(M, device=dev)
        f = lambda: w8.w8_rmsnorm_quant(x, gm, 1e-6, q=q, scale=s)
        byts = M * H * 3 + H * 2 + M * 4
    elif case == "silu_mul_quant":
        M, I = 4096, 12288
        x = rnd(M, 2 * I)
        q = torch.empty(M, I, dtype=torch.float8_e4m3fn, device=dev); s = torch.empty(M, device=dev)
        f = lambda: w8.w8_silu_mul_quant(x, q=q, scale=s)
        byts = M * I * 5 + M * 4
    elif case == "qk_norm_rope":
        T, Hq, Hkv, D = 16384, 32, 8, 128
        x = rnd(T, (Hq + 2 * Hkv) * D)
        qw = (torch.rand(D, device=dev, generator=g) + 0.5).to(torch.bfloat16); kw = qw.clone()
        pos = torch.randint(0, 8192, (T,), device=dev, generator=g)
        ang = torch.rand(8192, D // 2, device=dev, generator=g) * 6.283
        table = torch.cat([ang.cos(), ang.sin()], dim=1).float()
        f = lambda: w8.w8_qk_norm_rope(x, Hq, Hkv, D, qw, kw, table, pos, out=x)
        byts = T * (Hq + Hkv) * D * 4 + T * D * 4 + T * 8
    elif case in ("gemm_fp8", "gemm_int8", "gemm_block"):
        K, N, M = (4096, 24576, 8) if case != "gemm_block" else (5120, 51200, 8)
        fmt = {"gemm_fp8": 0, "gemm_int8": 1, "gemm_block": 2}[case]
        wb = rnd(N, K, scale=0.02)
        if fmt == 2:
            Wq, sW = w8.w8_quant_weight_block(wb)
            A, sA = w8.w8_quant_per_token(rnd(M, K), w8.W8_Q_FP8, group=128)
        else:
            qf = w8.W8_Q_INT8 if fmt == 1 else w8.W8_Q_FP8
            Wq, sW = w8.w8_quant_per_token(wb, qf)
            A, sA = w8.w8_quant_per_token(rnd(M, K), qf)
        del wb
        out = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        ws = w8.Workspace(dev)
        f = lambda: w8.w8_gemm(fmt, A, sA, Wq, sW, out=out, workspace=ws)
        byts = N * K + sW.numel() * 4 + M * K + sA.numel() * 4 + M * N * 2
        flops = 2 * M * N * K
    elif case == "grouped":
        E, N, K, M, top = 128, 1536, 2048, 4, 8
        wb = rnd(E * N, K, scale=0.02)
        Wq, sW = w8.w8_quant_per_token(wb, w8.W8_Q_FP8); del wb
        choice = torch.stack([torch.randperm(E, device=dev, generator=g)[:top] for _ in range(M)]).flatten()
        counts = torch.bincount(choice, minlength=E)
        off = torch.zeros(E + 1, dtype=torch.int32, device=dev); off[1:] = torch.cumsum(counts, 0).to(torch.int32)
        A, sA = w8.w8_quant_per_token(rnd(M * top, K), w8.W8_Q_FP8)
        out = torch.empty(M * top, N, dtype=torch.bfloat16, device=dev)
        ws = w8.Workspace(dev)
        f = lambda: w8.w8_grouped_gemm(0, A, sA, Wq.view(E, N, K), sW.view(E, N), off, max_tokens_per_expert=M,
                                       out=out, workspace=ws)
        used = int((counts > 0).sum().item())
        byts = used * N * (K + 4) + M * top * (K + 4) + M * top * N * 2
        flops = 2 * M * top * N * K
    elif case == "pair_prefill":
        M, K, N = 4096, 4096, 24576
        A, sA = w8.w8_quant_per_token(rnd(M, K), w8.W8_Q_FP8)
        Wq, sW = w8.w8_quant_per_token(rnd(N, K, scale=0.02), w8.W8_Q_FP8)
        out = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        ws = w8.Workspace(dev)
        f = lambda: w8.w8_gemm(0, A, sA, Wq, sW, out=out, workspace=ws)
        byts = M * K + N * K + (M + N) * 4 + M * N * 2
        flops = 2 * M * N * K
    else:
        raise SystemExit("unknown kernel case %r (one of: %s)" % (case, ", ".join(KERNEL_CASES)))
    return f, byts, flops


def _flush_l2(dev):
    import torch
    # write a buffer larger than L2 so the next launch reads its inputs from HBM
    torch.empty(256 << 20, dtype=torch.uint8, device=dev).fill_(1)


def run_kernel_case(case):
    """One hot-path kernel on its profiling-sized case (kernel_case), launched three times
    with a write larger than the L2 before each (for `ncu -k <kernel> -s 2 -c 1`)."""
    import torch
    from bit_quantized_gemm_token_b200 import w8
    if case not in KERNEL_CASES:
        raise SystemExit("unknown kernel case %r (one of: %s)" % (case, ", ".join(KERNEL_CASES)))
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(0)
    g = torch.Generator(device=dev); g.manual_seed(5)
    f, _, _ = kernel_case(case, dev, g)
    for _ in range(3):
        _flush_l2(dev)
        torch.cuda.synchronize()
        f()
        torch.cuda.synchronize()
    assert w8.w8_device_status(1) == 0
    print(json.dumps({"kernel_case": case, "launches": 3}))


def time_kernels(dev, peak, tflops_peak, reps=7):
    """Each hot-path kernel alone on its profiling-sized case (kernel_case): the median of
    `reps` launches, each timed with CUDA events on the launching stream after a write
    larger than the L2; HBM fraction (algorithmic bytes / time over the measured copy
    peak) and, for the contractions, the tensor fraction of the bf16 peak times 2 (fp8 and
    int8 run at twice the bf16 rate)."""
    import torch
    g = torch.Generator(device=dev); g.manual_seed(5)
    res = {}
    for case in KERNEL_CASES:
        f, byts, flops = kernel_case(case, dev, g)
        f()
        torch.cuda.synchronize()
        s = torch.cuda.current_stream()
        ts = []
        for _ in range(reps):
            _flush_l2(dev)
            e0 = torch.cuda.Event(enable_timing=True); e1 = torch.cuda.Event(enable_timing=True)
            e0.record(s); f(); e1.record(s)
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1) * 1e3)
        us = sorted(ts)[len(ts) // 2]
        r = {"us": round(us, 2), "GB/s": round(byts / (us * 1e-6) / 1e9, 1),
             "hbm_frac": round(byts / (us * 1e-6) / 1e9 / peak, 4), "bytes": byts}
        if flops and tflops_peak:
            r["TFLOP/s"] = round(flops / (us * 1e-6) / 1e12, 1)
            r["tensor_frac"] = round(flops / (us * 1e-6) / 1e12 / (2 * tflops_peak), 4)
        res[case] = r
        del f
        torch.cuda.empty_cache()
    return res


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--detail", action="store_true", help="also time every (shape, M) GEMM alone")
    ap.add_argument("--path", default="pair", choices=["pair", "linear"],
                    help="per layer: quantizer + GEMM calls (pair) or w8_linear (fused where it can)")
    ap.add_argument("--single", default="", help="KxN: time one shape only (profiling case)")
    ap.add_argument("--m", type=int, default=32)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip timing the other kernels (qk-norm/rope, grouped, the per-kernel table)")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-table", action="store_true", help="skip the per-(format, shape, M) decode table")
    ap.add_argument("--kernel", default="", help="run one kernel on its profiling case instead (for ncu): " +
                    ", ".join(KERNEL_CASES))
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--ref-seconds", type=float, default=3.0)
    args = ap.parse_args()
    if args.kernel:
        run_kernel_case(args.kernel)
        return
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
