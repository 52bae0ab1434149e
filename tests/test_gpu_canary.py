"""Out-of-bounds write detection without a sanitizer: every output buffer of
every entry point is the middle of a larger allocation whose guard regions
before and after hold a fixed byte pattern; after the call (at ragged shapes
that end tiles, groups and K slices mid-way) the guards must be untouched.
Outputs are also pre-filled, so a write that lands inside the buffer but at
the wrong place is caught by the parity tests, and a missing write by the
canary fill surviving where the oracle has a value."""
import numpy as np
import pytest
import torch

import weight_only_int4_quantize_b200 as w4
from weight_only_int4_quantize_b200 import synth

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA GPU")]

DEV = "cuda:0"
GUARD = 4096  # bytes on each side
PATTERN = 0x5A


class Guarded:
    """A tensor of `shape` and `dtype` inside a byte buffer with guards."""

    def __init__(self, shape, dtype):
        n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        self.raw = torch.full((GUARD + n + GUARD,), PATTERN, dtype=torch.uint8, device=DEV)
        self.n = n
        self.t = self.raw[GUARD:GUARD + n].view(dtype).view(shape)

    def check(self, what):
        torch.cuda.synchronize()
        head = self.raw[:GUARD]
        tail = self.raw[GUARD + self.n:]
        assert bool((head == PATTERN).all()), f"{what}: write before the buffer"
        assert bool((tail == PATTERN).all()), f"{what}: write after the buffer"


@pytest.mark.parametrize("sym", [False, True])
def test_quantize_outputs_guarded(sym):
    n, k = 301, 640
    w = synth.normal_weight(n, k, 0.02, seed=1).to(DEV)
    qw = Guarded((n, k // 8), torch.int32)
    sc = Guarded((n, k // 128), torch.int16)
    zr = None if sym else Guarded((n, k // 128), torch.int16)
    w4.lib().w4_quantize_pack(w.data_ptr(), n, k, 128, int(sym), None, 0.9, qw.t.data_ptr(),
                              sc.t.data_ptr(), None if zr is None else zr.t.data_ptr(),
                              torch.cuda.current_stream().cuda_stream)
    for g, name in ((qw, "qweight"), (sc, "scales"), (zr, "zeros")):
        if g is not None:
            g.check(name)
    rows = Guarded((n,), torch.float32)
    rows.t.fill_(0.8)
    qw2 = Guarded((n, k // 8), torch.int32)
    sc2 = Guarded((n, k // 128), torch.int16)
    zr2 = None if sym else Guarded((n, k // 128), torch.int16)
    assert w4.lib().w4_quantize_pack_rows(
        w.data_ptr(), n, k, 128, int(sym), None, rows.t.data_ptr(), qw2.t.data_ptr(),
        sc2.t.data_ptr(), None if zr2 is None else zr2.t.data_ptr(),
        torch.cuda.current_stream().cuda_stream) == 0
    for g in (qw2, sc2, zr2, rows):
        if g is not None:
            g.check("quantize rows")


# (M, N, K, flags): both decode kernels, the forced chunked decode, the
# prefill GEMM with 128/256-row tiles and with the cluster split of K.
LINEAR_CASES = [
    (1, 333, 1024, w4.LINEAR_DECODE_STREAM), (7, 333, 1024, w4.LINEAR_DECODE_TILED),
    (3, 40, 2048, 0), (13, 77, 768, 0), (40, 130, 640, w4.LINEAR_FORCE_GEMV),
    (33, 200, 8192, 0), (130, 300, 1024, 0), (300, 520, 4096, 0), (64, 300, 17408, 0),
]


@pytest.mark.parametrize("m,n,k,flags", LINEAR_CASES)
def test_linear_output_guarded(m, n, k, flags):
    w = synth.normal_weight(n, k, 0.02, seed=2).to(DEV)
    qw, sc, zr = w4.quantize_pack(w, False)
    x = synth.normal_activations(m, k, seed=3).to(DEV)
    y = Guarded((m, n), torch.bfloat16)
    w4.w4a16_linear(x, qw, sc, zr, flags=flags, out=y.t)
    y.check(f"y M={m} N={n} K={k}")
    assert bool(torch.isfinite(y.t.float()).all())


def test_batched_and_w4a8_outputs_guarded():
    items, guards = [], []
    for i, (n, k) in enumerate([(77, 1024), (300, 2048), (5, 128), (130, 6144)]):
        w = synth.normal_weight(n, k, 0.02, seed=10 + i).to(DEV)
        qw, sc, zr = w4.quantize_pack(w, False)
        x = synth.normal_activations(5, k, seed=20 + i).to(DEV)
        y = Guarded((5, n), torch.bfloat16)
        items.append((x, qw, sc, zr, y.t))
        guards.append(y)
    for flags in (w4.LINEAR_DECODE_STREAM, w4.LINEAR_DECODE_TILED):
        w4.w4a16_linear_batched(items, 5, flags)
        for y in guards:
            y.check("batched decode y")
    a8 = []
    for (x, qw, sc, zr, _y), y in zip(items, guards):
        m, k = x.shape
        xq = Guarded((m, k), torch.int8)
        xs = Guarded((m, k // 128), torch.int32)
        sx = Guarded((m,), torch.float32)
        assert w4.lib().w4_quantize_act_int8(x.data_ptr(), m, k, xq.t.data_ptr(), xs.t.data_ptr(),
                                             sx.t.data_ptr(),
                                             torch.cuda.current_stream().cuda_stream) == 0
        for g in (xq, xs, sx):
            g.check("int8 activations")
        a8.append((xq.t, xs.t, sx.t, qw, sc, zr, y.t))
    w4.w4a8_linear_batched(a8, 5)
    for y in guards:
        y.check("W4A8 y")


def test_scoring_outputs_guarded():
    x = synth.student_t_calibration(200, 640, seed=30).to(DEV)
    w = synth.normal_weight(300, 640, 0.02, seed=31).to(DEV)
    al, sh = synth.alpha_grid(4), synth.shrink_grid(3)
    al32 = np.ascontiguousarray(al, dtype=np.float32)
    sh32 = np.ascontiguousarray(sh, dtype=np.float32)
    sse = Guarded((1, 4, 3), torch.float64)
    arg = Guarded((2, 4), torch.int32)
    ws = Guarded((w4.awq_workspace_bytes(200, 300, 640, 4, 3),), torch.uint8)
    st = w4.lib().awq_score_grid(x.data_ptr(), 200, w.data_ptr(), 300, 640, 128, 0,
                                 al32.ctypes.data, 4, sh32.ctypes.data, 3, None, 1,
                                 sse.t.data_ptr(), arg.t.data_ptr(), ws.t.data_ptr(), ws.n,
                                 torch.cuda.current_stream().cuda_stream)
    assert st == 0
    for g, name in ((sse, "sse"), (arg, "argmins"), (ws, "workspace")):
        g.check(name)
    rows_sse = Guarded((3, 300), torch.float64)
    choice = Guarded((300,), torch.int32)
    rows = Guarded((300,), torch.float32)
    cws = Guarded((w4.clip_rows_workspace_bytes(200, 300, 640, 3),), torch.uint8)
    st = w4.lib().awq_clip_search_rows(x.data_ptr(), 200, w.data_ptr(), 300, 640, 128, 0, None,
                                       sh32.ctypes.data, 3, rows_sse.t.data_ptr(),
                                       choice.t.data_ptr(), rows.t.data_ptr(), cws.t.data_ptr(),
                                       cws.n, torch.cuda.current_stream().cuda_stream)
    assert st == 0
    for g, name in ((rows_sse, "row sse"), (choice, "choice"), (rows, "ratios"), (cws, "workspace")):
        g.check(name)


@pytest.mark.parametrize("ahead", [True, False])
def test_block_scoring_outputs_guarded(ahead):
    """Block-level losses and search: the losses, the choices and the whole
    workspace between guards, at a ragged token count (partial row tiles and
    causal tiles cut mid-way) on a small block."""
    cfg = {"hidden": 256, "heads": 4, "kv_heads": 2, "head_dim": 64, "ffn": 384, "eps": 1e-6,
           "rope_theta": 1e4}
    t = 70
    blk = {k: v.to(DEV) for k, v in synth.block_of_shape(cfg, 900).items()}
    nxt = {k: v.to(DEV) for k, v in synth.block_of_shape(cfg, 950).items()} if ahead else None
    x = synth.block_input(t, cfg["hidden"], seed=901).to(DEV)
    al = synth.alpha_grid(20)[[2, 9, 16]]
    sh = synth.shrink_grid(10)[[0, 4]]
    need = w4.block_workspace_bytes(t, cfg)
    ws = Guarded((need,), torch.uint8)
    losses = Guarded((3, 2), torch.float64)
    c = w4.BlockConfig(**cfg)
    import ctypes
    bi = w4._block_weights(blk, x)
    bn = w4._block_weights(nxt, x)
    al32, sh32 = np.ascontiguousarray(al), np.ascontiguousarray(sh)
    st = torch.cuda.current_stream().cuda_stream
    assert w4.lib().awq_block_scoring_losses(
        ctypes.byref(c), x.data_ptr(), t, ctypes.byref(bi),
        None if bn is None else ctypes.byref(bn), 0, al32.ctypes.data, 3, sh32.ctypes.data, 2, 0,
        -1, losses.t.data_ptr(), ws.t.data_ptr(), need, st) == 0
    losses.check("block losses")
    ws.check("block workspace (losses)")
    assert bool(torch.isfinite(losses.t).all())
    choice = Guarded((11,), torch.int32)
    sl = Guarded((4 * 3 + 7 * 2,), torch.float64)
    assert w4.lib().awq_block_search(
        ctypes.byref(c), x.data_ptr(), t, ctypes.byref(bi),
        None if bn is None else ctypes.byref(bn), al32.ctypes.data, 3, sh32.ctypes.data, 2, 1,
        choice.t.data_ptr(), sl.t.data_ptr(), ws.t.data_ptr(), need, st) == 0
    choice.check("block choices")
    sl.check("block search losses")
    ws.check("block workspace (search)")
    ch = choice.t.cpu().numpy()
    assert ((ch[:4] >= 0) & (ch[:4] < 3)).all() and ((ch[4:] >= 0) & (ch[4:] < 2)).all()
