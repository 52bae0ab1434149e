"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every function include/w4.h declares, and rejects bad arguments with the
documented status codes before touching the device."""
import ctypes
import os
import re

import pytest

import weight_only_int4_quantize_b200 as w4

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "w4.h")


@pytest.fixture(scope="module")
def L():
    if not os.path.exists(w4.LIB_PATH):
        from weight_only_int4_quantize_b200 import build
        build.build()
    return w4.lib()


def _declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\**\s+\**(\w+)\s*\(", src, flags=re.M)))


def test_exports_every_declared_function(L):
    names = _declared_functions()
    assert {"w4_quantize_pack", "w4a16_linear", "awq_score_grid", "w4_awq_scales",
            "w4_awq_workspace_bytes", "w4_status_string", "w4_device_error"} <= set(names)
    for n in names:
        assert hasattr(L, n), f"libw4.so does not export {n}"


def test_status_strings_and_version(L):
    for code in range(8):
        assert L.w4_status_string(code)
    assert L.w4_abi_version() == 1


A = 0x10000  # an aligned fake device address: validation runs before any device call
B = 0x20000


def test_quantize_validation(L):
    q = L.w4_quantize_pack
    assert q(None, 4, 128, 128, 0, None, 1.0, A, A, A, None) == 1       # NULL weight
    assert q(A, 4, 128, 128, 0, None, 1.0, A, A, None, None) == 1       # asym needs zeros
    assert q(A, 4, 128, 128, 1, None, 1.0, A, A, A, None) == 1          # sym forbids zeros
    assert q(A, 4, 128, 128, 0, None, 0.0, A, A, A, None) == 1          # shrink out of range
    assert q(A, 4, 128, 128, 0, None, 1.5, A, A, A, None) == 1
    assert q(A, 4, 128, 64, 0, None, 1.0, A, A, A, None) == 4           # group != 128
    assert q(A, 4, 100, 128, 0, None, 1.0, A, A, A, None) == 2          # K % 128
    assert q(A, 0, 128, 128, 0, None, 1.0, A, A, A, None) == 2          # N < 1
    assert q(A + 2, 4, 128, 128, 0, None, 1.0, A, A, A, None) == 3      # misaligned
    assert q(A, 4, 128, 128, 0, A + 4, 1.0, A, A, A, None) == 3         # misaligned s


def test_linear_validation(L):
    f = L.w4a16_linear
    assert f(None, 1, A, A, None, 8, 128, 128, B, 0, None) == 1
    assert f(A, 1, A, A, None, 8, 128, 128, B, 0x100, None) == 1        # unknown flag
    assert f(A, 1, A, A, None, 8, 128, 128, B, 0x3, None) == 1          # both forced paths
    assert f(A, 0, A, A, None, 8, 128, 128, B, 0, None) == 2
    assert f(A, 1, A, A, None, 8, 130, 128, B, 0, None) == 2
    assert f(A, 1, A, A, None, 8, 128, 32, B, 0, None) == 4
    assert f(A, 100, A, A, None, 8, 128, 128, B, 0x1, None) == 4        # GEMV beyond 64 rows
    assert f(A, 1, A, A, None, 8, 128, 128, B + 8, 0, None) == 3
    assert f(A, 1, A, A, None, 8, 128, 128, B, 0x30, None) == 1        # both decode kernels
    assert f(A, 1, A, A, None, 8, 128, 128, B, 0x12, None) == 1        # stream + prefill
    assert f(A, 9, A, A, None, 8, 128, 128, B, 0x10, None) == 4        # stream beyond 8 rows
    assert f(A, 65, A, A, None, 8, 128, 128, B, 0x20, None) == 4       # tiled beyond 64 rows


def test_linear_batched_validation(L):
    import weight_only_int4_quantize_b200 as w4
    f = L.w4a16_linear_batched
    it = (w4.LinearItem * 1)(w4.LinearItem(A, A, A, None, 8, 128, B))
    assert f(None, 1, 1, 128, 0, None) == 1
    assert f(it, 1, 1, 128, 0x1, None) == 1                            # not a batched flag
    assert f(it, 1, 1, 128, 0x30, None) == 1                           # both decode kernels
    assert f(it, 1, 9, 128, 0x10, None) == 4                           # stream beyond 8 rows
    assert f(it, 1, 1, 64, 0, None) == 4                               # group != 128


def test_awq_validation(L):
    f = L.awq_score_grid
    al = (ctypes.c_float * 2)(0.0, 0.5)
    sh = (ctypes.c_float * 2)(1.0, 0.9)
    bad_sh = (ctypes.c_float * 2)(1.0, 1.2)
    seg_bad = (ctypes.c_int64 * 3)(0, 100, 256)   # interior offset not a multiple of 16
    seg_ok = (ctypes.c_int64 * 3)(0, 128, 256)
    need = L.w4_awq_workspace_bytes(64, 256, 256, 2, 2, 2)
    assert need > 0
    base = (A, 64, B, 256, 256, 128, 0, al, 2, sh, 2)
    assert f(*base, None, 1, A, A, A, need, None) != 5  # reaches the device (no GPU here) or OK
    assert f(*base, seg_bad, 2, A, A, A, need, None) == 2
    assert f(*base, None, 2, A, A, A, need, None) == 1            # n_seg > 1 needs offsets
    assert f(*base, seg_ok, 2, A, A, A, 16, None) == 5            # workspace too small
    assert f(*base, seg_ok, 2, A, A, A + 16, need, None) == 3     # workspace not 256-aligned
    assert f(A, 64, B, 256, 256, 128, 0, al, 2, bad_sh, 2, None, 1, A, A, A, need, None) == 1
    assert f(A, 64, B, 256, 256, 128, 0, al, 0, sh, 2, None, 1, A, A, A, need, None) == 4
    assert L.w4_selftest_bounded_wait(10, None) == 1              # limit below 1 ms


def test_binding_fails_loudly_without_library(monkeypatch):
    monkeypatch.setattr(w4, "_LIB", None)
    monkeypatch.setattr(w4, "LIB_PATH", "/nonexistent/libw4.so")
    with pytest.raises(RuntimeError, match="no CPU fallback"):
        w4.lib()


def test_clip_rows_validation(L):
    import ctypes
    import numpy as np
    f = L.awq_clip_search_rows
    r = np.array([1.0, 0.9], np.float32)
    rp = r.ctypes.data
    big = 1 << 40
    assert f(None, 4, A, 8, 128, 128, 0, None, rp, 2, A, A, None, A, big, None) == 1
    assert f(A, 4, A, 8, 128, 64, 0, None, rp, 2, A, A, None, A, big, None) == 4     # group
    assert f(A, 4, A, 8, 128, 128, 0, None, rp, 0, A, A, None, A, big, None) == 4    # no grid
    assert f(A, 4, A, 8, 100, 128, 0, None, rp, 2, A, A, None, A, big, None) == 2    # K % 128
    bad = np.array([1.0, 1.5], np.float32)
    assert f(A, 4, A, 8, 128, 128, 0, None, bad.ctypes.data, 2, A, A, None, A, big, None) == 1
    assert f(A + 2, 4, A, 8, 128, 128, 0, None, rp, 2, A, A, None, A, big, None) == 3
    assert f(A, 4, A, 8, 128, 128, 0, None, rp, 2, A, A, None, None, 0, None) == 5   # workspace
    need = L.w4_clip_rows_workspace_bytes(4, 8, 128, 2)
    assert need > 0
    assert f(A, 4, A, 8, 128, 128, 0, None, rp, 2, A, A, None, A, need - 1, None) == 5
    assert f(A, 4, A, 8, 128, 128, 0, None, rp, 2, A, A, None, A + 16, need, None) == 3
    q = L.w4_quantize_pack_rows
    assert q(A, 4, 128, 128, 0, None, None, A, A, A, None) == 1                       # no ratios
    assert q(A, 4, 128, 128, 0, None, A + 2, A, A, A, None) == 3                      # misaligned
    assert q(A, 4, 128, 128, 1, None, A, A, A, A, None) == 1                          # sym + zeros
    assert q(A, 4, 128, 64, 0, None, A, A, A, A, None) == 4                           # group


def test_bench_and_entry_scripts_compile():
    """The driver runs these files directly: they must at least compile."""
    import py_compile
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    for name in ("bench.py", "__graft_entry__.py"):
        py_compile.compile(os.path.join(root, name), doraise=True)


def test_w4a8_validation(L):
    import weight_only_int4_quantize_b200 as w4
    q = L.w4_quantize_act_int8
    assert q(None, 1, 128, A, A, A, None) == 1
    assert q(A, 0, 128, A, A, A, None) == 2
    assert q(A, 1, 100, A, A, A, None) == 2
    assert q(A + 2, 1, 128, A, A, A, None) == 3
    f = L.w4a8_linear
    assert f(None, A, A, 1, A, A, None, 8, 128, 128, B, 0, None) == 1
    assert f(A, A, A, 17, A, A, None, 8, 128, 128, B, 0, None) == 4      # > 16 rows
    assert f(A, A, A, 1, A, A, None, 8, 128, 64, B, 0, None) == 4        # group
    assert f(A, A, A, 1, A, A, None, 8, 128, 128, B, 0x1, None) == 1     # not a W4A8 flag
    assert f(A, A, A, 1, A, A, None, 8, 130, 128, B, 0, None) == 2       # K % 128
    assert f(A, A + 4, A, 1, A, A, None, 8, 128, 128, B, 0, None) == 3   # misaligned xsum
    it = (w4.A8Item * 2)(w4.A8Item(A, A, A, A, A, None, 8, 128, B),
                         w4.A8Item(A, A, A, A, A, A, 8, 128, B))
    assert L.w4a8_linear_batched(it, 2, 1, 128, 0, None) == 1             # mixed symmetry


def test_binding_refuses_missized_companion_tensors(monkeypatch):
    """The C ABI takes bare pointers; the binding checks the shapes of every
    companion tensor before any call (CPU tensors here: the C library is
    replaced by a stub that must not be reached)."""
    import torch
    import weight_only_int4_quantize_b200 as w4

    class NoCall:
        def __getattr__(self, name):
            raise AssertionError(f"{name} reached with mis-sized inputs")

    monkeypatch.setattr(w4, "_cuda", lambda t, dtype, name: t)
    monkeypatch.setattr(w4, "lib", lambda: NoCall())
    x = torch.zeros(4, 256, dtype=torch.bfloat16)
    qw = torch.zeros(8, 32, dtype=torch.int32)
    sc = torch.zeros(8, 2, dtype=torch.int16)
    with pytest.raises(ValueError):
        w4.w4a16_linear(x, qw, torch.zeros(8, 3, dtype=torch.int16))
    with pytest.raises(ValueError):
        w4.w4a16_linear(x, qw, sc, torch.zeros(7, 2, dtype=torch.int16))
    with pytest.raises(ValueError):
        w4.w4a16_linear(x, qw, sc, out=torch.zeros(4, 9, dtype=torch.bfloat16))
    with pytest.raises(ValueError):
        w4.linear_items([(x, qw, sc, None, torch.zeros(4, 8, dtype=torch.bfloat16))], m=5)
    with pytest.raises(ValueError):
        w4.linear_items([(x, qw, sc, None, torch.zeros(3, 8, dtype=torch.bfloat16))])
    xq = torch.zeros(4, 256, dtype=torch.int8)
    with pytest.raises(ValueError):
        w4.w4a8_linear(xq, torch.zeros(4, 3, dtype=torch.int32), torch.zeros(4), qw, sc)
    with pytest.raises(ValueError):
        w4.w4a8_linear(xq, torch.zeros(4, 2, dtype=torch.int32), torch.zeros(5), qw, sc)
    with pytest.raises(ValueError):
        w4.a8_items([(xq, torch.zeros(4, 2, dtype=torch.int32), torch.zeros(4), qw,
                      torch.zeros(8, 1, dtype=torch.int16), None,
                      torch.zeros(4, 8, dtype=torch.bfloat16))])
    with pytest.raises(ValueError):
        w4.quantize_pack_items([(torch.zeros(8, 256, dtype=torch.bfloat16), torch.zeros(255),
                                 1.0, qw, sc, None)])
    with pytest.raises(ValueError):
        w4.quantize_pack(torch.zeros(8, 256, dtype=torch.bfloat16), False,
                         awq_s=torch.zeros(128))
    with pytest.raises(ValueError):
        w4.awq_clip_search_rows(x, torch.zeros(8, 128, dtype=torch.bfloat16), [1.0], False)


def _block_structs(align_off=0, missing=None):
    cfg = w4.BlockConfig(**w4.QWEN3_1P7B_BLOCK)
    fields = {f[0]: A + 0x1000 * i + align_off for i, f in enumerate(w4._BlockWeights._fields_)}
    if missing:
        fields[missing] = None
    return cfg, w4._BlockWeights(**fields)


def test_block_validation(L):
    """awq_block_scoring_losses / awq_block_search / w4_block_workspace_bytes
    reject bad arguments before any device call."""
    import numpy as np
    by = ctypes.byref
    cfg, blk = _block_structs()
    ws_need = L.w4_block_workspace_bytes(by(cfg), 256)
    assert ws_need > 0
    # the workspace grows with T (the attention scores are heads x T^2)
    assert L.w4_block_workspace_bytes(by(cfg), 512) > ws_need
    assert L.w4_block_workspace_bytes(by(cfg), 0) == 0
    assert L.w4_block_workspace_bytes(None, 256) == 0
    bad = w4.BlockConfig(**dict(w4.QWEN3_1P7B_BLOCK, head_dim=96))
    assert L.w4_block_workspace_bytes(by(bad), 256) == 0
    al = np.array([0.0, 0.5], np.float32)
    sh = np.array([1.0, 0.9], np.float32)
    pa, ps = al.ctypes.data, sh.ctypes.data

    def score(cfg_=cfg, x=A, t=256, blk_=blk, nxt=None, group=0, alphas=pa, na=2, shrinks=ps,
              nr=2, only=-1, out=B, ws=A, wsb=None):
        return L.awq_block_scoring_losses(
            None if cfg_ is None else by(cfg_), x, t, None if blk_ is None else by(blk_),
            None if nxt is None else by(nxt), group, alphas, na, shrinks, nr, 0, only, out, ws,
            ws_need if wsb is None else wsb, None)

    assert score(out=None) == 1                 # no output
    assert score(group=4) == 1                  # group out of range
    assert score(group=0, only=3) == 1          # o is not in qkv
    assert score(group=2, only=6) == 1          # down is not in gate_up
    assert score(cfg_=None) == 1
    assert score(blk_=None) == 1
    _, blk_missing = _block_structs(missing="k_norm")
    assert score(blk_=blk_missing) == 1         # a missing gain
    assert score(nxt=blk_missing) == 1          # the next block checked too
    assert score(cfg_=bad) == 2                 # head_dim
    assert score(cfg_=w4.BlockConfig(**dict(w4.QWEN3_1P7B_BLOCK, kv_heads=3))) == 2
    assert score(t=0) == 2
    assert score(t=8193) == 2
    assert score(na=0) == 4
    assert score(na=65) == 4
    assert score(shrinks=np.array([1.0, 1.5], np.float32).ctypes.data) == 1
    assert score(alphas=np.array([0.0, np.nan], np.float32).ctypes.data) == 1
    _, blk_mis = _block_structs(align_off=8)
    assert score(blk_=blk_mis) == 3             # misaligned weights
    assert score(x=A + 8) == 3                  # misaligned input
    assert score(out=B + 8) == 3                # misaligned losses
    assert score(wsb=ws_need - 1) == 5          # workspace too small
    assert score(ws=A + 128) == 3               # workspace not 256-byte aligned

    def search(choice=B, losses=None, **kw):
        return L.awq_block_search(by(cfg), A, 256, by(blk), None, pa, 2, ps, 2, 0, choice, losses,
                                  A, kw.get("wsb", ws_need), None)

    assert search(choice=None) == 1
    assert search(choice=B + 4) == 3
    assert search(losses=B + 8) == 3
    assert search(wsb=16) == 5


def test_bench_traffic_captures_match_sources():
    """bench.py reports a kernel's DRAM traffic from an ncu capture only while
    the kernel's source is the one captured (its digest); a kernel changed
    without a new capture would report null."""
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    for kernel, cap in bench.TRAFFIC_CAPTURES.items():
        assert bench.source_digest(cap["source"]) == cap["digest"], (
            f"{kernel}: {cap['source']} changed since its traffic capture")
        assert 0.3 < cap["ratio"] < 1.5, kernel
    e = bench.roofline_entry("gemv_w4a16", "hbm", 4000.0, 6535.7, "GB/s", "measured", 1e9, 0.5)
    assert e["frac"] == 4000.0 / 6535.7 and e["traffic"] == bench.TRAFFIC_CAPTURES[
        "gemv_w4a16"]["ratio"] * 1e9
