"""The C-ABI library loads, exports every entry point the header declares, and
rejects bad arguments on the host before touching a GPU (no GPU needed)."""
import ctypes
import os
import re

import pytest

import mixture_experts_routed_moe_b200 as moe
from mixture_experts_routed_moe_b200 import _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FAKE = 1 << 20  # a 256-byte aligned non-null address; never dereferenced by the host checks


@pytest.fixture(scope="module")
def L():
    _build.build()
    return moe.lib()


def header_functions():
    text = open(os.path.join(ROOT, "include", "moe_b200.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(L):
    names = header_functions()
    assert set(names) == set(moe.EXPORTS)
    for n in names:
        assert hasattr(L, n), n
    nm = os.popen(f"nm -D --defined-only {moe.LIB_PATH}").read()
    for n in names:
        assert re.search(rf"\bT {n}\b", nm), n


def test_version_and_status_strings(L):
    assert L.moe_version() >= 100
    for code in moe.STATUS:
        assert moe.status_string(code)
    assert "UE8M0" in moe.status_string(-3)


def shape(**kw):
    d = dict(T=64, H=128, I=256, E=8, k=2, wdtype="bf16", path="auto")
    d.update(kw)
    return moe.make_shape(**d)


@pytest.mark.parametrize("bad", [dict(H=100), dict(I=96), dict(E=0), dict(E=1025), dict(k=0), dict(k=9),
                                 dict(T=-1), dict(wdtype=7), dict(path=9), dict(H=0), dict(act=3)])
def test_invalid_shapes_rejected(L, bad):
    s = shape(**bad)
    assert L.moe_workspace_size(ctypes.byref(s)) == 0
    lay = moe.MoeWorkspaceLayout()
    assert L.moe_workspace_query(ctypes.byref(s), ctypes.byref(lay)) == -1
    r = L.moe_forward(ctypes.byref(s), FAKE, FAKE, FAKE, FAKE, FAKE, None, None, FAKE, FAKE, 1 << 40, None)
    assert r == -1


@pytest.mark.parametrize("H,I", [(128, 64), (192, 256), (64, 64)])
def test_bf16_64_aligned_sizes_are_unsupported_not_invalid(L, H, I):
    """bf16 layers with H, I multiples of 64 but not of 128 are valid requests
    this build does not run: MOE_ERR_UNSUPPORTED, not MOE_ERR_INVALID_ARG;
    the same sizes with e4m3 experts are invalid (FP8 needs 128-wide blocks)."""
    s = shape(H=H, I=I)
    r = L.moe_forward(ctypes.byref(s), FAKE, FAKE, FAKE, FAKE, FAKE, None, None, FAKE, FAKE, 1 << 40, None)
    assert r == -2
    assert L.moe_workspace_size(ctypes.byref(s)) == 0
    s = shape(H=H, I=I, wdtype="e4m3")
    r = L.moe_forward(ctypes.byref(s), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 40, None)
    assert r == -1


def test_workspace_layout_is_consistent(L):
    for path, bm in (("prefill", 128), ("decode", 1)):
        s = shape(T=300, E=60, k=4, H=2048, I=1408, path=path)
        lay = moe.workspace_layout(s)
        assert lay.bm == bm and lay.path == moe.PATH[path]
        total = moe.workspace_size(s)
        assert total == lay.total
        A = 300 * 4
        assert lay.m_rows >= A + (min(60, A) * (bm - 1) if bm > 1 else 0)
        offs = [lay.status, lay.hdr, lay.cnt, lay.mt_base, lay.row_src, lay.slot_row, lay.h, lay.y]
        assert offs == sorted(offs) and all(o % 256 == 0 for o in offs)
        assert lay.y + lay.m_rows * 2048 * 2 <= total
        # x rows staged expert-major for the tensor-core GEMMs on both paths
        # (tile-padded on PREFILL, one row per assignment on DECODE)
        assert lay.xa != 2 ** 64 - 1 and lay.h - lay.xa >= lay.m_rows * 2048 * 2


def test_e4m3_workspace_layouts(L):
    """e4m3 PREFILL: x codes per permuted row; e4m3 DECODE: x codes once per
    token (T rows), then h codes and scales per assignment row."""
    T, H, I, E, k = 16, 7168, 2048, 256, 8
    pre = moe.workspace_layout(shape(T=T, H=H, I=I, E=E, k=k, wdtype="e4m3", path="prefill"))
    dec = moe.workspace_layout(shape(T=T, H=H, I=I, E=E, k=k, wdtype="e4m3", path="decode"))
    assert dec.bm == 1 and dec.m_rows == T * k and pre.bm == 128
    # decode: xa holds T rows of H codes, xs T rows of H/128 fp32 scales
    assert dec.xs - dec.xa >= T * H and dec.xs - dec.xa < T * H + 1024
    assert dec.h - dec.xs >= T * (H // 128) * 4
    # prefill: one row of codes per permuted row
    assert pre.xs - pre.xa >= pre.m_rows * H
    for lay in (pre, dec):
        assert lay.hs - lay.h >= lay.m_rows * I  # e4m3 h codes
        assert lay.y + lay.m_rows * H * 2 <= lay.total


def test_auto_path_choice(L):
    """The decode-stage switch: the DECODE path while T*k <= 32E (bf16),
    T*k <= 2E (FP4) or 2*T*k <= E (e4m3), the grouped GEMMs beyond; the
    boundary cases included."""
    D, P = moe.PATH["decode"], moe.PATH["prefill"]
    assert moe.workspace_layout(shape(T=16, H=2048, I=1408, E=60, k=4)).path == D
    assert moe.workspace_layout(shape(T=480, H=2048, I=1408, E=60, k=4)).path == D  # 1920 = 32E
    assert moe.workspace_layout(shape(T=481, H=2048, I=1408, E=60, k=4)).path == P
    assert moe.workspace_layout(shape(T=8192, H=2048, I=768, E=128, k=8)).path == P
    assert moe.workspace_layout(shape(T=16, H=7168, I=2048, E=256, k=8, wdtype="e4m3")).path == D  # 128 = E/2
    assert moe.workspace_layout(shape(T=17, H=7168, I=2048, E=256, k=8, wdtype="e4m3")).path == P
    assert moe.workspace_layout(shape(T=64, H=7168, I=2048, E=256, k=8, wdtype="e2m1")).path == D  # 512 = 2E
    assert moe.workspace_layout(shape(T=65, H=7168, I=2048, E=256, k=8, wdtype="e2m1")).path == P
    assert moe.workspace_layout(shape(T=4096, E=60, k=4, wdtype="e4m3")).path == P


def test_scale_format_error_and_host_errors(L):
    s = shape(wdtype="e4m3")
    # FP8 experts without UE8M0 scales: refused loudly
    r = L.moe_forward(ctypes.byref(s), FAKE, FAKE, FAKE, FAKE, FAKE, None, None, FAKE, FAKE, 1 << 40, None)
    assert r == -3
    # e4m3 PREFILL with H not a multiple of 256: refused before any launch
    s = shape(wdtype="e4m3", path="prefill", H=384)
    r = L.moe_forward(ctypes.byref(s), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 40, None)
    assert r == -2
    s = shape()
    need = moe.workspace_size(s)
    r = L.moe_forward(ctypes.byref(s), FAKE, FAKE, FAKE, FAKE, FAKE, None, None, FAKE, FAKE, need - 1, None)
    assert r == -4
    r = L.moe_forward(ctypes.byref(s), None, FAKE, FAKE, FAKE, FAKE, None, None, FAKE, FAKE, need, None)
    assert r == -1
    r = L.moe_forward(ctypes.byref(s), FAKE + 8, FAKE, FAKE, FAKE, FAKE, None, None, FAKE, FAKE, need, None)
    assert r == -1  # misaligned x
    r = L.moe_forward(ctypes.byref(s), FAKE, FAKE, FAKE, FAKE, FAKE, None, None, FAKE, FAKE + 16, need, None)
    assert r == -1  # misaligned workspace
    # empty input: nothing to do, nothing enqueued
    s0 = shape(T=0)
    assert L.moe_forward(ctypes.byref(s0), None, None, None, None, None, None, None, None, None, 0, None) == 0
    # bad timing-event count
    ev = (ctypes.c_void_p * 3)()
    assert L.moe_forward_timed(ctypes.byref(s), FAKE, FAKE, FAKE, FAKE, FAKE, None, None, FAKE, FAKE, need, None,
                               ev, 3) == -1


def test_route_host_errors(L):
    assert L.moe_route(FAKE, 4, 0, 1, FAKE, FAKE, None) == -1
    assert L.moe_route(FAKE, 4, 8, 9, FAKE, FAKE, None) == -1
    assert L.moe_route(FAKE, -1, 8, 2, FAKE, FAKE, None) == -1
    assert L.moe_route(None, 4, 8, 2, FAKE, FAKE, None) == -1
    assert L.moe_route(None, 0, 8, 2, None, None, None) == 0


def test_router_host_errors(L):
    # (x, w_router, T, H, E, k, logits, idx, w, stream)
    assert L.moe_router(FAKE, FAKE, 4, 128, 257, 2, None, FAKE, FAKE, None) == -1  # E > 256
    assert L.moe_router(FAKE, FAKE, 4, 100, 8, 2, None, FAKE, FAKE, None) == -1  # H not a multiple of 64
    assert L.moe_router(FAKE, FAKE, 4, 128, 8, 9, None, FAKE, FAKE, None) == -1  # k > E
    assert L.moe_router(FAKE + 8, FAKE, 4, 128, 8, 2, None, FAKE, FAKE, None) == -1  # misaligned x
    assert L.moe_router(None, FAKE, 4, 128, 8, 2, None, FAKE, FAKE, None) == -1
    assert L.moe_router(None, None, 0, 128, 8, 2, None, None, None, None) == 0  # T == 0: nothing to do


def test_test_hooks_validate_and_reset(L):
    assert L.moe_set_test_hooks(2, 0) == -1
    assert L.moe_set_test_hooks(0, 999_999) == -1  # below 1 ms
    assert L.moe_set_test_hooks(0, 60_000_000_001) == -1
    assert L.moe_set_test_hooks(1, 5_000_000) == 0
    assert L.moe_set_test_hooks(0, 0) == 0  # back to the defaults
    with pytest.raises(moe.MoeError):
        moe.set_test_hooks(wait_limit_ns=10)


def test_missing_library_fails_loudly(monkeypatch):
    monkeypatch.setattr(moe, "_lib", None)
    monkeypatch.setattr(moe, "LIB_PATH", "/nonexistent/libmoe_b200.so")
    with pytest.raises(ImportError):
        moe.lib()


def test_product_code_never_touches_the_oracle():
    pkg = os.path.join(ROOT, "mixture_experts_routed_moe_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                src = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(from|import)\s+oracle|moe_oracle|oracle/", src, flags=re.M), f


def test_binding_checks_tensor_arguments():
    """The binding refuses what the C ABI cannot see: wrong dtype, rank,
    layout or device (checked before anything reaches the library)."""
    import torch

    T, H, I, E, k = 4, 128, 128, 4, 2
    x = torch.zeros((T, H), dtype=torch.bfloat16)
    idx = torch.zeros((T, k), dtype=torch.int32)
    w = torch.zeros((T, k), dtype=torch.float32)
    wgu = torch.zeros((E, 2 * I, H), dtype=torch.bfloat16)
    wd = torch.zeros((E, H, I), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="x must be on a CUDA device"):
        moe.forward(x, idx, w, wgu, wd)
    with pytest.raises(ValueError, match="topk_idx: dtype"):
        moe._need(idx.long(), "topk_idx", (torch.int32,), 2)
    with pytest.raises(ValueError, match="x: 1-D"):
        moe._need(x[0], "x", (torch.bfloat16,), 2)
    with pytest.raises(ValueError, match="contiguous"):
        moe._need(wgu.transpose(1, 2), "w_gate_up", (torch.bfloat16,), 3)
    with pytest.raises(TypeError):
        moe._need(None, "x", (torch.bfloat16,), 2)
    with pytest.raises(ValueError, match="logits: dtype"):
        moe.route(torch.zeros((T, E), dtype=torch.float64), k)
    with pytest.raises(ValueError, match="x must be on a CUDA device"):
        moe.router(x, torch.zeros((E, H), dtype=torch.bfloat16), k)


def test_binding_checks_sizes_before_any_launch():
    """Every tensor's sizes are checked against the layer that x, topk_idx and
    w_gate_up define, so no kernel can read or write past an allocation
    (checked on the host, before the device check and before the library)."""
    import torch

    T, H, I, E, k = 4, 128, 128, 4, 2
    bf = torch.bfloat16
    ok = dict(x=torch.zeros((T, H), dtype=bf), topk_idx=torch.zeros((T, k), dtype=torch.int32),
              topk_w=torch.zeros((T, k), dtype=torch.float32), w_gate_up=torch.zeros((E, 2 * I, H), dtype=bf),
              w_down=torch.zeros((E, H, I), dtype=bf))

    def call(**bad):
        a = dict(ok)
        a.update(bad)
        return moe.forward(**a)

    cases = [
        (dict(w_gate_up=torch.zeros((E, 2 * I, H + 128), dtype=bf)), "w_gate_up: shape"),
        (dict(w_gate_up=torch.zeros((E, 2 * I + 1, H), dtype=bf)), "2\\*I"),
        (dict(w_down=torch.zeros((E, H, 2 * I), dtype=bf)), "w_down: shape"),
        (dict(w_down=torch.zeros((E + 1, H, I), dtype=bf)), "w_down: shape"),
        (dict(topk_w=torch.zeros((T, k + 1), dtype=torch.float32)), "topk_w: shape"),
        (dict(topk_idx=torch.zeros((T + 1, k), dtype=torch.int32)), "topk_idx: shape"),
        (dict(out=torch.zeros((T, H - 8), dtype=bf)), "out: shape"),
        (dict(sw_gate_up=torch.zeros((E, 2, 1), dtype=torch.uint8)), "bf16 experts"),
        (dict(workspace=torch.zeros((8, 8), dtype=torch.uint8)), "workspace: 2-D"),
    ]
    for bad, msg in cases:
        with pytest.raises(ValueError, match=msg):
            call(**bad)
    # e4m3 experts: the UE8M0 block grids must match the weights
    f8 = torch.float8_e4m3fn
    e4 = dict(w_gate_up=torch.zeros((E, 2 * I, H), dtype=f8), w_down=torch.zeros((E, H, I), dtype=f8))
    with pytest.raises(ValueError, match="sw_gate_up: shape"):
        call(**e4, sw_gate_up=torch.zeros((E, 2 * I // 128, H // 128 + 1), dtype=torch.uint8),
             sw_down=torch.zeros((E, H // 128, I // 128), dtype=torch.uint8))
    with pytest.raises(ValueError, match="sw_down: shape"):
        call(**e4, sw_gate_up=torch.zeros((E, 2 * I // 128, H // 128), dtype=torch.uint8),
             sw_down=torch.zeros((E, I // 128, H // 128 + 1), dtype=torch.uint8))
    with pytest.raises(ValueError, match="w_down: dtype"):
        call(w_gate_up=torch.zeros((E, 2 * I, H), dtype=f8))
    # well-formed arguments get as far as the device check
    with pytest.raises(ValueError, match="x must be on a CUDA device"):
        call()
    with pytest.raises(ValueError, match="w_router: shape"):
        moe.router(ok["x"], torch.zeros((E, H + 64), dtype=bf), k)
    with pytest.raises(ValueError, match="topk_w: shape"):
        moe.route(torch.zeros((T, E), dtype=torch.float32), k, topk_w=torch.zeros((T, k + 1)))


def test_binding_requires_one_device():
    """A tensor on another device than x is refused (the library launches on
    the current device only)."""
    import torch

    dev = torch.device("cuda", 0)
    with pytest.raises(ValueError, match="w_down is on cpu"):
        moe._same_device(dev, w_down=torch.zeros(1))
    with pytest.raises(ValueError, match="on a CUDA device"):
        moe._same_device(torch.device("cpu"))
    moe._same_device(dev, out=None)  # absent tensors are fine


def test_pipeline_needs_two_batches_in_flight():
    """MoEPipeline overlaps the copies of neighbouring batches with the
    compute only with at least two buffer sets; fewer is refused before any
    device work."""
    with pytest.raises(ValueError):
        moe.MoEPipeline(None, 16, depth=1)
