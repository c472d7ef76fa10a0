"""On-device variant selector: writes the static dispatch table.

    python -m quantized_linear_gemm_b200.sweep [--configs decode,block,prefill] [--formats ...]
        [--with-quant] [--out PATH] [--inc]

For every (format, token bucket, N, K) of the Qwen3 decode / prefill shapes
this enumerates the variant space - Swap-AB or Standard, tile_n, split_k,
the reduction mode, ring depth and launch mode - times each candidate under
CUDA-graph replay with weight copies rotated so that every call reads its
weights from HBM, and keeps the fastest.  It replaces the offline autotuner
of the techfeed.io summary of the Helion blog (section "オートチューニングの仕組み":
an LLM-seeded tree search) by exhaustive search: the space is small and
discrete.

The result is a text table (one line per key, the format that
lq_load_dispatch_table reads) and, with --inc, the compiled-in table
csrc/dispatch_table.inc.  Correctness of every variant is covered by the
test suite; the sweep only measures.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import sys
import time

import torch

from . import inputs, lq

PKG = os.path.dirname(os.path.abspath(__file__))
TABLE_TXT = os.path.join(PKG, "dispatch_table.txt")
TABLE_INC = os.path.join(PKG, "csrc", "dispatch_table.inc")
L2_BYTES = 126 * 2 ** 20
FMT_NAMES = {lq.FP8_DYNAMIC: "fp8_dynamic", lq.W8A8_INT8: "w8a8_int8", lq.BLOCK_FP8: "block_fp8",
             lq.BLOCK_FP8_UE8M0: "block_fp8_ue8m0"}


def keys_for(groups):
    keys = []
    if "decode" in groups:
        for fmt in (lq.FP8_DYNAMIC, lq.W8A8_INT8):
            for (K, N) in inputs.QWEN3_8B.values():
                for M in inputs.DECODE_M:
                    keys.append((fmt, M, N, K))
    if "block" in groups:
        for (K, N) in inputs.QWEN3_32B.values():
            for M in inputs.DECODE_M:
                keys.append((lq.BLOCK_FP8, M, N, K))
    if "prefill" in groups:
        for fmt in (lq.FP8_DYNAMIC, lq.W8A8_INT8, lq.BLOCK_FP8):
            for layer in ("gate_up", "down"):
                K, N = inputs.QWEN3_32B[layer]
                for M in inputs.PREFILL_M:
                    keys.append((fmt, M, N, K))
    if "ue8m0" in groups:   # Block_FP8 with UE8M0 scales (the tensor core's block-scaled MMA)
        for (K, N) in inputs.QWEN3_32B.values():
            for M in inputs.DECODE_M:
                keys.append((lq.BLOCK_FP8_UE8M0, M, N, K))
    if "ue8m0-prefill" in groups:
        for layer in ("gate_up", "down"):
            K, N = inputs.QWEN3_32B[layer]
            for M in inputs.PREFILL_M:
                keys.append((lq.BLOCK_FP8_UE8M0, M, N, K))
    return keys


PAIRS = 74   # CTA pairs resident at once on a B200 (148 SMs)


def candidates(fmt, M, N, K):
    T = -(-K // 128)
    out = []

    def add(**kw):
        out.append(lq.make_variant(**kw))

    if M <= 64:
        tns = [16, 32] if M <= 32 else [32, 64]   # M = 24, 32 also as two 16-token tiles
        for tn in tns:
            for S in (1, 2, 4, 8, 16):
                if S > T:
                    continue
                per = -(-T // S)
                for st in sorted({2, min(per, 3), min(per, 4), min(per, 5), min(per, 6), min(per, 8), min(per, 12)}):
                    if st < 2:
                        continue
                    for pdl in (1, 2):
                        add(swap_ab=1, tile_n=tn, split_k=S, stages=st, reduce=2, pdl=pdl)
            for S in (32, 64):
                if S <= T // 2:
                    add(swap_ab=1, tile_n=tn, split_k=S, stages=2, reduce=1, pdl=2)
                    add(swap_ab=1, tile_n=tn, split_k=S, stages=2, reduce=0, pdl=2)
            for S in (3, 5, 6):   # split counts that fill the SMs where powers of two leave a partial wave
                if S <= T:
                    per = -(-T // S)
                    for st in sorted({min(per, 3), min(per, 4), min(per, 6)}):
                        if st >= 2:
                            add(swap_ab=1, tile_n=tn, split_k=S, stages=st, reduce=1, pdl=2)
    if M >= 16:
        tns = (64, 128) if fmt == lq.BLOCK_FP8 else (64, 128, 256)   # fp32-scale Block_FP8: up to 128
        for tn in tns:
            for S in (1, 2, 4, 8):
                if S > T:
                    continue
                for st in (3, 4, 6, 0):
                    for pdl in (1, 2):
                        add(swap_ab=0, tile_n=tn, split_k=S, stages=st, reduce=2, pdl=pdl)
            if -(-M // 128) * -(-N // tn) < 148:   # few tiles: split counts between the powers of two
                for S in (3, 5, 6, 7):
                    if S <= T:
                        for st in (3, 4, 0):
                            add(swap_ab=0, tile_n=tn, split_k=S, stages=st, reduce=1, pdl=2)
            if fmt in (lq.BLOCK_FP8, lq.BLOCK_FP8_UE8M0) and tn == 128:   # Block_FP8 on CTA pairs (256 x 128 tiles)
                for st in (4, 6, 0):
                    for pdl in (1, 2):
                        add(swap_ab=0, tile_n=tn, split_k=1, stages=st, pdl=pdl, persistent=2)
            if fmt in (lq.FP8_DYNAMIC, lq.W8A8_INT8):   # persistent CTAs and CTA pairs (one split)
                for st in (3, 4, 0):
                    for pdl in (1, 2):
                        add(swap_ab=0, tile_n=tn, split_k=1, stages=st, pdl=pdl, persistent=1)
                        if tn >= 128:
                            add(swap_ab=0, tile_n=tn, split_k=1, stages=st, pdl=pdl, persistent=2)
                            add(swap_ab=0, tile_n=tn, split_k=1, stages=st, pdl=pdl, persistent=3)
            # CTA pairs with Split-K where the 256-row tiles alone leave pairs idle
            pair_ok = tn == 128 if fmt in (lq.BLOCK_FP8, lq.BLOCK_FP8_UE8M0) else tn >= 128
            tiles = -(-M // 256) * -(-N // tn)
            if pair_ok and tiles < PAIRS:
                for S in range(2, 9):
                    if S <= T and tiles * S <= 3 * PAIRS:
                        for st in (3, 4, 0):
                            add(swap_ab=0, tile_n=tn, split_k=S, stages=st, reduce=0, pdl=2, persistent=2)
    return out


class Shape:
    """Device buffers of one (fmt, M, N, K) with enough weight copies that
    more than 2x L2 is streamed between two reads of one copy."""

    def __init__(self, fmt, M, N, K, device, with_quant=False):
        self.fmt, self.M, self.N, self.K = fmt, M, N, K
        self.with_quant = with_quant and fmt not in (lq.BLOCK_FP8, lq.BLOCK_FP8_UE8M0)
        name = FMT_NAMES[fmt]
        w = inputs.weights(N, K, seed=inputs.stable_seed("sweep-W", N, K)).to(device)
        x = inputs.activations(M, K, seed=inputs.stable_seed("sweep-A", M, K)).to(device)
        self.x = x
        if fmt == lq.BLOCK_FP8:
            qb, sb = lq.quant_weight_block128(w)
            self.qa, self.sa = lq.quant_per_token_group128(x)
        elif fmt == lq.BLOCK_FP8_UE8M0:
            qb, sb = lq.quant_weight_block128_ue8m0(w)
            self.qa, self.sa = lq.quant_per_token_group128_ue8m0(x)
        else:
            qb, sb = lq.quant_per_token(name, w)
            self.qa, self.sa = lq.quant_per_token(name, x)
        del w
        wbytes = N * K
        self.copies = max(2, min(64, math.ceil(2 * L2_BYTES / wbytes) + 1))
        self.W = [(qb, sb)] + [(qb.clone(), sb.clone()) for _ in range(self.copies - 1)]
        self.C = torch.empty((M, N), dtype=torch.bfloat16, device=device)
        self.bytes = lq.Problem(fmt, M, N, K).bytes
        self.flops = 2 * M * N * K

    def time_us(self, v, stream, calls=None, replays=8):
        calls = calls or self.copies
        try:
            lq.reserve_workspace(stream.device.index, lq.workspace_bytes(self.fmt, self.M, self.N, self.K, v))
            with torch.cuda.stream(stream):
                for i in range(2):
                    qb, sb = self.W[i % self.copies]
                    lq.scaled_mm(self.fmt, self.qa, self.sa, qb, sb, C=self.C, variant=v, stream=stream)
            torch.cuda.synchronize()
        except lq.LQError:
            return None
        g = torch.cuda.CUDAGraph()
        name = FMT_NAMES[self.fmt]
        with torch.cuda.stream(stream):
            with torch.cuda.graph(g, stream=stream):
                for i in range(calls):
                    qb, sb = self.W[i % self.copies]
                    if self.with_quant:   # as in a decode step: the activations are quantized right before
                        lq.quant_per_token(name, self.x, self.qa, self.sa, stream=stream)
                    lq.scaled_mm(self.fmt, self.qa, self.sa, qb, sb, C=self.C, variant=v, stream=stream)
        g.replay()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(replays):
                g.replay()
            e1.record(stream)
        e1.synchronize()
        del g
        return 1e3 * e0.elapsed_time(e1) / (replays * calls)


def sweep(groups, device, log=sys.stderr, budget_s=None, with_quant=False, formats=None, ms=None):
    stream = torch.cuda.Stream(device=device)
    results = []
    t_start = time.time()
    for key in keys_for(groups):
        fmt, M, N, K = key
        if formats is not None and fmt not in formats:
            continue
        if ms is not None and M not in ms:
            continue
        sh = Shape(fmt, M, N, K, device, with_quant=with_quant)
        big = sh.flops > 2e11
        best = None
        tried = 0
        timed = []
        for v in candidates(fmt, M, N, K):
            us = sh.time_us(v, stream, calls=(4 if big else None), replays=(3 if big else 8))
            tried += 1
            if us is not None:
                timed.append((us, v))
            if us is not None and (best is None or us < best[0]):
                best = (us, v)
        # re-time the winner (and the runner-up choice is implicit) to reduce noise
        us = sh.time_us(best[1], stream, calls=(4 if big else None), replays=(5 if big else 20))
        gbs = sh.bytes / (us * 1e-6) / 1e9
        tf = sh.flops / (us * 1e-6) / 1e12
        rec = dict(fmt=FMT_NAMES[fmt], M=M, N=N, K=K, us=round(us, 3), gbs=round(gbs, 1), tflops=round(tf, 2),
                   variant=best[1].as_dict(), candidates=tried,
                   top=[dict(us=round(u, 3), variant=v.as_dict()) for u, v in sorted(timed, key=lambda x: x[0])[:5]])
        results.append(rec)
        print(json.dumps(rec), file=log, flush=True)
        del sh
        torch.cuda.empty_cache()
        if budget_s and time.time() - t_start > budget_s:
            print("sweep: time budget reached", file=log)
            break
    return results


def m_bucket(M):
    for p in (1, 2, 4, 8, 16, 24, 32):
        if M <= p:
            return p
    b = 64
    while b < M:
        b *= 2
    return b


def write_table(results, path):
    lines = ["# dispatch table written by quantized_linear_gemm_b200.sweep (measured on B200)",
             "# fmt m_bucket N K swap_ab split_k tile_n stages reduce pdl   # us GB/s TFLOP/s"]
    for r in results:
        v = r["variant"]
        lines.append(f"{r['fmt']} {m_bucket(r['M'])} {r['N']} {r['K']} {v['swap_ab']} {v['split_k']} {v['tile_n']} "
                     f"{v['stages']} {v['reduce']} {v['pdl']} {v.get('persistent', 0)}   "
                     f"# {r['us']} {r['gbs']} {r['tflops']}")
    with open(path, "w") as f:
        f.write("\n".join(lines) + "\n")


def merge_table(base_path, new_path, out_path):
    """The entries of base_path with those of new_path added; an entry of
    new_path replaces the base entry of the same (fmt, m_bucket, N, K)."""
    def entries(path):
        out = []
        for line in open(path):
            body = line.split("#")[0].split()
            if body:
                out.append((tuple(body[:4]), line.rstrip("\n")))
        return out
    new = entries(new_path)
    keys = {k for k, _ in new}
    kept = [ln for k, ln in entries(base_path) if k not in keys]
    head = [ln.rstrip("\n") for ln in open(base_path) if ln.startswith("#")]
    with open(out_path, "w") as f:
        f.write("\n".join(head + kept + [ln for _, ln in new]) + "\n")


def write_inc(txt_path, inc_path):
    fmt_id = {"fp8_dynamic": 0, "w8a8_int8": 1, "block_fp8": 2, "block_fp8_ue8m0": 3}
    rows = []
    for line in open(txt_path):
        line = line.split("#")[0].split()
        if not line:
            continue
        f, mb, n, k, sw, sk, tn, st, rd, pdl = line[:10]
        pers = line[10] if len(line) > 10 else "0"
        rows.append(f"    {{{fmt_id[f]}, {mb}, {n}, {k}, {{{sw}, {sk}, {tn}, {st}, {rd}, {pdl}, {pers}}}}},")
    body = "\n".join(rows) if rows else "    {-1, 0, 0, 0, {0, 1, 64, 2, 1, 1, 0}},   // placeholder (never matches)"
    with open(inc_path, "w") as f:
        f.write("// Compiled-in dispatch table: (format, token bucket, N, K) -> variant.\n"
                "// Generated by quantized_linear_gemm_b200/sweep.py from dispatch_table.txt\n"
                "// (measured best variants on B200).  Keys not listed use the heuristic.\n"
                "// fields: fmt, m_bucket, N, K, {swap_ab, split_k, tile_n, stages, reduce, pdl, persistent}\n"
                "static const TableEntry kDefaultTable[] = {\n" + body + "\n};\n"
                f"static const size_t kDefaultTableSize = {len(rows)};\n")


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--configs", default="decode,block,prefill")
    ap.add_argument("--out", default=TABLE_TXT)
    ap.add_argument("--json", default=None, help="also write the measurements as JSON lines here")
    ap.add_argument("--inc", action="store_true", help="regenerate csrc/dispatch_table.inc from --out")
    ap.add_argument("--inc-only", action="store_true", help="only regenerate the .inc from an existing table")
    ap.add_argument("--budget-s", type=float, default=None)
    ap.add_argument("--formats", default=None, help="comma-separated subset, e.g. fp8_dynamic")
    ap.add_argument("--ms", default=None, help="comma-separated subset of M values, e.g. 256")
    ap.add_argument("--merge", default=None, metavar="TABLE",
                    help="merge the measured entries into TABLE (same key: replaced) and write the result to --out")
    ap.add_argument("--with-quant", action="store_true",
                    help="time each candidate after lq_quant_per_token, as the decode step runs it")
    a = ap.parse_args()
    if a.inc_only:
        write_inc(a.out, TABLE_INC)
        return
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    lq.init_device(0)
    lq.load_dispatch_table(None)
    fmts = None if a.formats is None else {lq.FORMATS[f] for f in a.formats.split(",")}
    ms = None if a.ms is None else {int(m) for m in a.ms.split(",")}
    res = sweep(set(a.configs.split(",")), device, budget_s=a.budget_s, with_quant=a.with_quant, formats=fmts, ms=ms)
    if a.merge:
        tmp = a.out + ".new"
        write_table(res, tmp)
        merge_table(a.merge, tmp, a.out)
        os.remove(tmp)
    else:
        write_table(res, a.out)
    if a.json:
        with open(a.json, "w") as f:
            for r in res:
                f.write(json.dumps(r) + "\n")
    if a.inc:
        write_inc(a.out, TABLE_INC)


if __name__ == "__main__":
    main()
