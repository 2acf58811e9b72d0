"""Offline variant sweep on the B200: for every (format, shape, M bucket) time the legal
GEMM variants (Swap-AB / Standard, tile width, Standard / Split-K / balanced partition,
K blocks per stage, CTAs per SM, pipeline depth) and write the fastest into the
per-shape table that w8_load_table reads.  This is the role of the per-shape
precomputed configs of the pages ("Helion nel backend vLLM ...", paragraphs 3-4), with
an exhaustive search over a small space instead of their autotuner.

Each candidate is checked before it is timed: its output must equal the reference
variant's bit for bit for INT8 (int32 accumulators) and within the GEMM tolerance for
the fp8 formats.  Timing: a CUDA graph of (activation quant, GEMM) pairs, as in use,
with programmatic dependent launch, rotating over enough weight copies to exceed 3x
the L2; CUDA events on the capturing stream.  A GEMM's cost depends on the kernel
before it (how its tail overlaps this one's start), so each candidate is timed in
context: every pair of the shape under test follows a pair of the shape that precedes
it in the layer's order (qkv -> o -> gate_up -> down -> qkv), and the candidate with the
lowest time for the two pairs wins.  A first pass puts the built-in choice in front; a
second pass re-times the best few behind the first pass's winners.

    python -m bit_quantized_gemm_token_b200.sweep [--out PATH] [--quick] [--formats 0,1,2]
                                                  [--families swap,bm64,decode,shipped]
"""
import argparse
import json
import os
import time

import torch

from . import w8

DENSE = [(4096, 6144), (4096, 4096), (4096, 24576), (12288, 4096)]
BLOCK = [(5120, 10240), (5120, 51200), (25600, 5120), (4096, 6144)]
MS = [1, 2, 4, 8, 16, 32]
HERE = os.path.dirname(os.path.abspath(__file__))
DEFAULT_OUT = os.path.join(HERE, "tuning", "b200_table.txt")


def decode_estimate(M, N, K, bn, c):
    """Microseconds the built-in rule estimates for the decode form (the same model as
    the library's: HBM stream, one CTA's stream, its MMA chain, the cluster exchange)."""
    kbs = -(-K // 128)
    kb = -(-kbs // c)
    t = max(N * K / 6.5e6, bn * kb * 128 / 54e3, kb * 4 * 0.084)
    return t + (0.25 * c if c > 1 else 0.0)


def decode_candidates(fmt, M, N, K, sms=148, keep=10):
    """Decode-form variants (FP8 / INT8, M <= 64): the `keep` (tile, K chunks) pairs the
    model ranks best among those filling 60-100% of the SMs, each at the default pipeline
    depth and at a deeper one."""
    if fmt >= 2 or M > 64:
        return []
    kbs = -(-K // 128)
    pairs = []
    for bn in range(64, 257, 16):
        tiles = -(-N // bn)
        for c in range(1, 9):
            if c > kbs or tiles * c > sms or tiles * c < 0.6 * sms:
                continue
            pairs.append((decode_estimate(M, N, K, bn, c), bn, c))
    pairs.sort()
    out = []
    m8 = (M + 7) // 8 * 8
    for _, bn, c in pairs[:keep]:
        stage = (m8 + bn) * 128
        deep = min(8, 196608 // stage)
        for st in sorted({0, deep}):
            out.append(w8.decode_variant(bn, c, stages=st, l2ahead=0))
    return out


def shipped_variant(fmt, M, N, K):
    """The variant the table shipped with the package resolves to (0 if none)."""
    best = None
    if os.path.exists(DEFAULT_OUT):
        for line in open(DEFAULT_OUT):
            f = line.split("#")[0].split()
            if len(f) != 5:
                continue
            r = [int(x) for x in f[:4]] + [int(f[4], 16)]
            if r[0] == fmt and r[1] == N and r[2] == K and r[3] >= M and (best is None or r[3] < best[3]):
                best = r
    return best[4] if best else 0


def candidates(fmt, M, N, K, quick=False, families=("swap", "bm64", "decode")):
    block = fmt >= 2
    out = []
    if "decode" in families:
        out += decode_candidates(fmt, M, N, K)
    if "fused" in families and fmt < 2:
        # the decode form with the activation quantizer inside (w8_linear, one kernel)
        out += [v | w8.W8_V_FUSED for v in decode_candidates(fmt, M, N, K)]
    if "shipped" in families:
        v = shipped_variant(fmt, M, N, K)
        if v:
            out.append(v)
    if "mid" in families:
        # token counts past the decode form: 256 x 256 tiles on CTA pairs, and the one-CTA
        # Standard loops with 128 x 128 / 128 x 256 tiles whole, split over K or balanced
        for stages in (0, 4, 6):
            out.append(w8.variant(False, 1, 256, stages=stages, pair=True))
        for split in (2, 4, 8):
            for stages in (0, 4):
                out.append(w8.variant(False, split, 256, stages=stages, pair=True))
        for bn in (128, 256):
            for kind, arg in [("split", 1), ("split", 2), ("split", 4), ("split", 8), ("stream", 1), ("stream", 2)]:
                if kind == "stream":
                    out.append(w8.variant(False, 1, bn, stream=True, cps=arg))
                else:
                    out.append(w8.variant(False, arg, bn))
    if "swap" not in families:
        return _legal(fmt, M, N, K, out)
    bns = [b for b in (16, 32, 64) if b >= min(M, 64)][:2]
    for bn in bns:
        parts = [("stream", 1), ("stream", 2)] + [("split", s) for s in (1, 2, 4, 8, 16)] + \
                [("cluster", s) for s in (2, 4, 8)]
        for kind, arg in parts:
            for kps in (1, 2):
                for stages in ((0,) if quick else (0, 2, 3, 4, 5, 6)):
                    if kind == "stream":
                        v = w8.variant(True, 1, bn, stream=True, stages=stages, kps=kps, cps=arg)
                    else:
                        v = w8.variant(True, arg, bn, stages=stages, kps=kps, cluster=(kind == "cluster"))
                    out.append(v)
    if not block and "bm64" in families:
        # Standard form, 64-row token tile, weights in the MMA's N slot
        for bn in (128, 256):
            parts = [("stream", 1), ("split", 1), ("split", 2), ("split", 4), ("split", 8), ("cluster", 2), ("cluster", 4),
                     ("cluster", 8)]
            for kind, arg in parts:
                for kps in (1, 2):
                    for stages in ((0,) if quick else (0, 2, 3, 4)):
                        if kind == "stream":
                            v = w8.variant(False, 1, bn, stream=True, stages=stages, kps=kps, cps=arg, bm64=True)
                        else:
                            v = w8.variant(False, arg, bn, stages=stages, kps=kps, cluster=(kind == "cluster"), bm64=True)
                        out.append(v)
        # the same with the parallel fixup of split tiles
        for bn in (128, 256):
            for kind, arg in [("stream", 1), ("split", 2), ("split", 4), ("split", 8)]:
                for kps in (1, 2):
                    for stages in ((0,) if quick else (0, 3, 4, 5)):
                        if kind == "stream":
                            v = w8.variant(False, 1, bn, stream=True, stages=stages, kps=kps, cps=1, bm64=True,
                                           pfix=True)
                        else:
                            v = w8.variant(False, arg, bn, stages=stages, kps=kps, bm64=True, pfix=True)
                        out.append(v)
    return _legal(fmt, M, N, K, out)


def _legal(fmt, M, N, K, out):
    legal = []
    for v in out:
        try:
            if v & w8.W8_V_FUSED:
                w8.w8_linear_resolve(fmt, M, N, K, v)
            else:
                w8.w8_gemm_resolve_variant(fmt, M, N, K, v)
            legal.append(v)
        except w8.W8Error:
            pass
    return sorted(set(legal))


class Problem:
    def __init__(self, fmt, N, K, ms, dev):
        self.fmt, self.N, self.K = fmt, N, K
        g = torch.Generator(device=dev)
        g.manual_seed(4321 + N + K + fmt)
        self.ncopy = max(2, -(-400_000_000 // (N * K)))
        qf = w8.W8_Q_INT8 if fmt == 1 else w8.W8_Q_FP8
        self.W = []
        for _ in range(self.ncopy):
            wb = (torch.randn(N, K, device=dev, generator=g) * 0.02).to(torch.bfloat16)
            if fmt >= 2:
                self.W.append(w8.w8_quant_weight_block(wb, ue8m0=(fmt == 3)))
            else:
                self.W.append(w8.w8_quant_per_token(wb, qf))
            del wb
        self.A, self.X = {}, {}
        self.qf = qf
        for M in ms:
            x = torch.randn(M, K, device=dev, generator=g).to(torch.bfloat16)
            self.X[M] = x
            self.A[M] = self.quant(M)
        self.ws = w8.Workspace(dev)
        self.dev = dev
        self.outs = {}

    def quant(self, M):
        A = self.A.get(M)
        q, s = (A if A is not None else (None, None))
        if self.fmt >= 2:
            return w8.w8_quant_per_token(self.X[M], w8.W8_Q_FP8, group=128, ue8m0=(self.fmt == 3), q=q, scale=s)
        return w8.w8_quant_per_token(self.X[M], self.qf, q=q, scale=s)

    def run(self, M, v, copy=0, out=None):
        A, sA = self.A[M]
        Wq, sW = self.W[copy]
        return w8.w8_gemm(self.fmt, A, sA, Wq, sW, out=out, variant=v, workspace=self.ws)

    def linear(self, M, v, copy=0, out=None):
        Wq, sW = self.W[copy]
        return w8.w8_linear(self.fmt, self.X[M], Wq, sW, out=out, variant=v, workspace=self.ws)

    def layer(self, M, v, copy, out):
        """One layer as used: the activation quantizer and the GEMM, or one kernel."""
        if v & w8.W8_V_FUSED:
            self.linear(M, v, copy, out)
        else:
            self.quant(M)
            self.run(M, v, copy, out)

    def check(self, M, v, ref_v):
        if v & w8.W8_V_FUSED:
            # the fused kernel against the two kernels with the same variant: the same bytes
            a = self.linear(M, v)
            b = self.linear(M, v & ~w8.W8_V_FUSED)
            torch.cuda.synchronize()
            return torch.equal(a, b)
        A, _ = self.A[M]
        if self.fmt == 1:
            a = w8.w8_gemm_i32_debug(A, self.W[0][0], variant=v, workspace=self.ws)
            b = w8.w8_gemm_i32_debug(A, self.W[0][0], variant=ref_v, workspace=self.ws)
            torch.cuda.synchronize()
            return torch.equal(a, b)
        a = self.run(M, v).float()
        b = self.run(M, ref_v).float()
        torch.cuda.synchronize()
        return bool(((a - b).abs().max() <= 2.0 ** -7 * b.abs().max() + 1e-3).item())

    def out(self, M):
        o = self.outs.get(M)
        if o is None:
            o = self.outs[M] = torch.empty((M, self.N), dtype=torch.bfloat16, device=self.dev)
        return o


def time_in_context(prev, pv, prob, M, v, reps=2):
    """Microseconds per (prev pair, tested pair): a CUDA graph of alternating (quant,
    GEMM) pairs, `prev` with variant pv in front of every pair of `prob` with v."""
    v = v | w8.W8_V_PDL
    pv = pv | w8.W8_V_PDL
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    for p, var in ((prev, pv), (prob, v)):
        p.ws.reserve(max(w8.w8_gemm_workspace_size(p.fmt, M, p.N, p.K, var & ~w8.W8_V_FUSED),
                         w8.w8_linear_workspace_size(p.fmt, M, p.N, p.K, var)))
    n = max(prev.ncopy, prob.ncopy)

    def body():
        for c in range(n):
            # as in use: the activation quantizer runs right before every GEMM (or inside it)
            prev.layer(M, pv, c % prev.ncopy, prev.out(M))
            prob.layer(M, v, c % prob.ncopy, prob.out(M))

    with torch.cuda.stream(s):
        body()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for _ in range(reps):
            body()
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    best = float("inf")
    for _ in range(3):
        with torch.cuda.stream(s):
            e0.record(s)
            g.replay()
            e1.record(s)
        torch.cuda.synchronize()
        best = min(best, e0.elapsed_time(e1) * 1e3 / (reps * n))
    del g
    return best


def default_variant(fmt, M):
    """The reference every candidate's output is checked against: Swap-AB, balanced."""
    bn = 16 if M <= 16 else 32 if M <= 32 else 64
    return w8.variant(True, 1, bn, stream=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--out", default=DEFAULT_OUT)
    ap.add_argument("--quick", action="store_true", help="default pipeline depths only")
    ap.add_argument("--formats", default="0,1,2")
    ap.add_argument("--families", default="swap,bm64,decode",
                    help="candidate families: swap (Swap-AB), bm64 (64-row token tile), decode, fused (decode form with "
                         "the quantizer inside, w8_linear), mid (CTA pairs "
                         "and one-CTA Standard loops for larger token counts), shipped (the current table's "
                         "entry)")
    ap.add_argument("--log", default="")
    ap.add_argument("--ms", default=",".join(str(m) for m in MS), help="token counts to sweep")
    ap.add_argument("--shapes", default="",
                    help="KxN,KxN,...: sweep these shapes instead of the format's default list (rows of the other "
                         "shapes are kept); in the layer order they run in")
    args = ap.parse_args()
    ms = [int(m) for m in args.ms.split(",")]
    only = [tuple(int(v) for v in sh.lower().split("x")) for sh in args.shapes.split(",")] if args.shapes else None
    families = tuple(args.families.split(","))
    # rows of formats not swept now are kept from the table being replaced
    kept = []
    fmts_swept = set()
    for f in args.formats.split(","):
        fmts_swept |= {2, 3} if int(f) == 2 else {int(f)}
    if os.path.exists(args.out):
        for line in open(args.out):
            f = line.split("#")[0].split()
            if len(f) != 5:
                continue
            swept_shape = only is None or (int(f[2]), int(f[1])) in only
            if int(f[0]) not in fmts_swept or int(f[3]) not in ms or not swept_shape:
                kept.append((int(f[0]), int(f[1]), int(f[2]), int(f[3]), int(f[4], 16)))
    os.environ["W8_TABLE"] = "none"
    w8.w8_clear_table()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    fmts = [int(f) for f in args.formats.split(",")]
    rows = []
    log = []
    t_start = time.time()
    top_n = 8
    for fmt in fmts:
        shapes = only if only else (BLOCK if fmt >= 2 else DENSE)
        probs = [Problem(fmt, N, K, ms, dev) for (K, N) in shapes]
        for M in ms:
            ref_v = default_variant(fmt, M)
            cands = []
            for prob in probs:
                ok = []
                for v in candidates(fmt, M, prob.N, prob.K, args.quick, families):
                    if prob.check(M, v, ref_v):
                        ok.append(v)
                    else:
                        log.append({"fmt": fmt, "N": prob.N, "K": prob.K, "M": M, "variant": hex(v), "error": "mismatch"})
                cands.append(ok)
            # pass 1: the built-in choice in front of every shape; pass 2: the best few
            # again, behind the pass-1 winners
            choice = [w8.w8_gemm_resolve_variant(fmt, M, p.N, p.K, w8.W8_VARIANT_AUTO) for p in probs]
            results = [None] * len(probs)
            for npass in (1, 2):
                front = list(choice)
                for i, prob in enumerate(probs):
                    prev = probs[i - 1]
                    pool = cands[i] if npass == 1 else [v for _, v in results[i][:top_n]]
                    res = sorted((time_in_context(prev, front[i - 1], prob, M, v), v) for v in pool)
                    results[i] = res
                    choice[i] = res[0][1]
            for i, prob in enumerate(probs):
                res = results[i]
                N, K = prob.N, prob.K
                best_us, best_v = res[0]
                base_us = [u for u, v in res if v == ref_v]
                rec = {"fmt": fmt, "N": N, "K": K, "M": M, "pair_us_in_context": round(best_us, 3),
                       "after": "%dx%d" % (probs[i - 1].K, probs[i - 1].N), "variant": hex(best_v),
                       "desc": w8.describe(best_v),
                       "default_us": round(base_us[0], 3) if base_us else None,
                       "top5": [(round(u, 2), hex(v)) for u, v in res[:5]]}
                log.append(rec)
                print(json.dumps(rec), flush=True)
                for f in ([2, 3] if fmt == 2 else [fmt]):
                    rows.append((f, N, K, M, best_v))
        del probs
        torch.cuda.empty_cache()
    rows += kept
    rows.sort(key=lambda r: (r[0], r[2], r[1], r[3]))
    os.makedirs(os.path.dirname(args.out), exist_ok=True)
    with open(args.out, "w") as fh:
        fh.write("# per-shape GEMM variant table for B200 (sm_100a), written by\n")
        fh.write("# python -m bit_quantized_gemm_token_b200.sweep; columns: fmt N K m_max variant\n")
        fh.write("# fmt 0 = FP8-dynamic, 1 = W8A8-INT8, 2/3 = Block-FP8 (fp32 / UE8M0 scales)\n")
        for r in rows:
            fh.write("%d %d %d %d 0x%x\n" % r)
    if args.log:
        with open(args.log, "w") as fh:
            json.dump(log, fh, indent=0)
    print("wrote %d entries to %s in %.0f s" % (len(rows), args.out, time.time() - t_start))


if __name__ == "__main__":
    main()
