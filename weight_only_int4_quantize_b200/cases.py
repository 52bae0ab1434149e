"""Runs one library call on a named shape, for profilers (ncu) and quick
timing.  Inputs are seeded and generated on the device.

    python -m weight_only_int4_quantize_b200.cases quantize --n 17408 --k 5120 [--sym]
    python -m weight_only_int4_quantize_b200.cases linear --m 8 --n 17408 --k 5120 [--sym] [--gemm]
    python -m weight_only_int4_quantize_b200.cases awq --m 2048 --n 1024 --k 2048 --na 20 --nr 10
    python -m weight_only_int4_quantize_b200.cases decode_batch --m 1 --blocks 4 [--a8]
    python -m weight_only_int4_quantize_b200.cases clip_rows --m 2048 --n 6144 --k 2048 --nr 10
    python -m weight_only_int4_quantize_b200.cases block --t 512 --na 2 [--group qkv] [--own]
    python -m weight_only_int4_quantize_b200.cases block --search --t 2048 --na 20 --nr 10

Each case captures --iters launches in one CUDA graph (so host launch
overhead does not count), replays it once to warm up, times one replay with
CUDA events and prints the mean time per launch and the algorithmic
throughput.  Back-to-back launches of one linear re-read the same weights:
for weights smaller than L2 this measures L2, not HBM.
"""
from __future__ import annotations

import argparse
import json

import torch

import weight_only_int4_quantize_b200 as w4
from weight_only_int4_quantize_b200 import synth


def _weights(n, k, seed, std=0.02):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    return (torch.randn(n, k, generator=g, device="cuda") * std).to(torch.bfloat16)


def _time(fn, iters, graph=True):
    """Mean device time per call: `iters` calls captured in one CUDA graph
    (no host launch overhead between them), replayed after a warm replay."""
    fn()
    torch.cuda.synchronize()
    if graph:
        g = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            with torch.cuda.graph(g, stream=s):
                for _ in range(iters):
                    fn()
        torch.cuda.current_stream().wait_stream(s)
        run = g.replay
        run()
    else:
        def run():
            for _ in range(iters):
                fn()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    run()
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / iters


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("case", choices=["quantize", "linear", "awq", "decode_batch", "clip_rows",
                                     "block"])
    ap.add_argument("--t", type=int, default=512, help="block: tokens entering the block")
    ap.add_argument("--group", default="qkv", help="block: linear group scored")
    ap.add_argument("--own", action="store_true",
                    help="block: loss at the block's own output (no look-ahead)")
    ap.add_argument("--search", action="store_true",
                    help="block: the screened search (na alphas x nr shrinks) instead of the "
                         "binary64 losses of one group")
    ap.add_argument("--blocks", type=int, default=4,
                    help="decode_batch: Qwen3-1.7B-shaped blocks (7 linears each) in one batch")
    ap.add_argument("--m", type=int, default=8)
    ap.add_argument("--n", type=int, default=4096)
    ap.add_argument("--k", type=int, default=4096)
    ap.add_argument("--sym", action="store_true")
    ap.add_argument("--gemm", action="store_true", help="force the tcgen05 prefill kernel")
    ap.add_argument("--gemv", action="store_true", help="force the decode kernel")
    ap.add_argument("--na", type=int, default=20)
    ap.add_argument("--nr", type=int, default=10)
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--copies", type=int, default=1,
                    help="linear: weight copies used in turn (working set above L2)")
    ap.add_argument("--pdl", action="store_true", help="programmatic dependent launch + static weights")
    ap.add_argument("--eager", action="store_true", help="time eager launches instead of a graph")
    ap.add_argument("--a8", action="store_true", help="decode_batch: W4A8 (int8 activations)")
    ap.add_argument("--kernel", choices=["auto", "stream", "tiled"], default="auto",
                    help="decode kernel (linear, decode_batch)")
    a = ap.parse_args()
    if a.case == "block":
        # Block-level losses of a.na alphas (shrink 1) of one group of a
        # Qwen3-1.7B-shaped block, binary64 (two block forwards per candidate).
        import numpy as np
        gi = {k: v.cuda() for k, v in synth.qwen_block(3).items()}
        gn = None if a.own else {k: v.cuda() for k, v in synth.qwen_block(4).items()}
        x = synth.block_input(a.t, 2048, seed=77).cuda()
        ws = torch.empty(w4.block_workspace_bytes(a.t), dtype=torch.uint8, device="cuda")
        al = synth.alpha_grid(20)[: a.na]
        one = np.array([1.0], np.float32)
        if a.search:
            sh = synth.shrink_grid(10)[: a.nr]
            ms = _time(lambda: w4.awq_block_search(x, gi, gn, al, sh, False, workspace=ws),
                       a.iters, False)
            n_c = 4 * a.na + 7 * a.nr
            print(json.dumps({"case": "block_search", "t": a.t, "candidates": n_c,
                              "lookahead": not a.own, "ms": ms, "ms_per_candidate": ms / n_c}))
            return
        ms = _time(lambda: w4.awq_block_scoring_losses(x, gi, gn, a.group, al, one, False,
                                                       workspace=ws), a.iters, False)
        print(json.dumps({"case": "block", "t": a.t, "group": a.group, "candidates": a.na,
                          "lookahead": not a.own, "ms": ms, "ms_per_candidate": ms / a.na}))
        return
    kflag = {"auto": 0, "stream": w4.LINEAR_DECODE_STREAM,
             "tiled": w4.LINEAR_DECODE_TILED}[a.kernel]
    w = _weights(a.n, a.k, 1)
    out = {"case": a.case, "m": a.m, "n": a.n, "k": a.k, "sym": a.sym}
    if a.case == "quantize":
        ms = _time(lambda: w4.quantize_pack(w, a.sym), a.iters, not a.eager)
        b = a.n * a.k * (2.5 + (2 if a.sym else 4) / 128)
        out.update(ms=ms, gbs=b / ms / 1e6)
    elif a.case == "linear":
        # --copies C: C packed copies of the weight, used in turn, so that a
        # working set above L2 is read from HBM.
        packs = [w4.quantize_pack(w, a.sym)]
        for c in range(1, a.copies):
            packs.append(w4.quantize_pack(_weights(a.n, a.k, 1 + c), a.sym))
        del w
        g = torch.Generator(device="cuda")
        g.manual_seed(2)
        x = torch.randn(a.m, a.k, generator=g, device="cuda").to(torch.bfloat16)
        y = torch.empty(a.m, a.n, dtype=torch.bfloat16, device="cuda")
        flags = (w4.LINEAR_FORCE_GEMM if a.gemm else 0) | (w4.LINEAR_FORCE_GEMV if a.gemv else 0)
        flags |= kflag
        if a.pdl:
            flags |= w4.LINEAR_PDL | w4.LINEAR_STATIC_WEIGHTS
        turn = [0]

        def run():
            qw, sc, zr = packs[turn[0] % len(packs)]
            turn[0] += 1
            w4.w4a16_linear(x, qw, sc, zr, flags=flags, out=y)
        ms = _time(run, a.iters * len(packs), not a.eager)
        out["copies"] = len(packs)
        b = a.n * a.k * (0.5 + (2 if a.sym else 4) / 128) + 2 * a.m * (a.k + a.n)
        out.update(ms=ms, gbs=b / ms / 1e6, tflops=2.0 * a.m * a.n * a.k / ms / 1e9,
                   kernel=a.kernel)
    elif a.case == "decode_batch":
        # a.blocks x 7 independent linears at a.m tokens through
        # w4a16_linear_batched (asymmetric), as one decode step would run them.
        del w
        items, byts = [], 0.0
        for bi in range(a.blocks):
            for li, (_name, k, n) in enumerate(synth.QWEN3_1P7B_BLOCK):
                wb = _weights(n, k, 100 + 7 * bi + li)
                qw, sc, zr = w4.quantize_pack(wb, False)
                del wb
                g = torch.Generator(device="cuda")
                g.manual_seed(200 + 7 * bi + li)
                x = torch.randn(a.m, k, generator=g, device="cuda").to(torch.bfloat16)
                y = torch.empty(a.m, n, dtype=torch.bfloat16, device="cuda")
                items.append((x, qw, sc, zr, y))
                byts += n * k * (0.5 + 4 / 128) + 2 * a.m * (k + n)
        flags = (w4.LINEAR_PDL | w4.LINEAR_STATIC_WEIGHTS if a.pdl else 0) | kflag
        if a.a8:  # W4A8: activations quantized once, outside the timed launches
            # (the activation tensors stay referenced: the item array holds
            # raw pointers only)
            acts = [w4.quantize_act_int8(x) for (x, *_r) in items]
            arr = w4.a8_items([(*q8, qw, sc, zr, y)
                               for q8, (x, qw, sc, zr, y) in zip(acts, items)])
            ms = _time(lambda: w4.w4a8_linear_batched(arr, a.m, flags), a.iters, not a.eager)
        else:
            arr = w4.linear_items(items)
            ms = _time(lambda: w4.w4a16_linear_batched(arr, a.m, flags), a.iters, not a.eager)
        out.update(ms=ms, gbs=byts / ms / 1e6, linears=len(items), a8=a.a8, kernel=a.kernel)
    elif a.case == "clip_rows":
        g = torch.Generator(device="cuda")
        g.manual_seed(3)
        x = (torch.randn(a.m, a.k, generator=g, device="cuda")).to(torch.bfloat16)
        sh = synth.shrink_grid(a.nr)
        ws = torch.empty(w4.clip_rows_workspace_bytes(a.m, a.n, a.k, a.nr), dtype=torch.uint8,
                         device="cuda")
        ms = _time(lambda: w4.awq_clip_search_rows(x, w, sh, a.sym, workspace=ws), a.iters, False)
        out.update(ms=ms, tflops=2.0 * a.m * a.n * a.k * a.nr / ms / 1e9)
    else:
        g = torch.Generator(device="cuda")
        g.manual_seed(3)
        x = (torch.randn(a.m, a.k, generator=g, device="cuda")).to(torch.bfloat16)
        al, sh = synth.alpha_grid(a.na), synth.shrink_grid(a.nr)
        ws = torch.empty(w4.awq_workspace_bytes(a.m, a.n, a.k, a.na, a.nr), dtype=torch.uint8,
                         device="cuda")
        ms = _time(lambda: w4.awq_score_grid(x, w, al, sh, a.sym, workspace=ws), a.iters, False)
        out.update(ms=ms, tflops=2.0 * a.m * a.n * a.k * a.na * a.nr / ms / 1e9)
    print(json.dumps(out))


if __name__ == "__main__":
    main()
