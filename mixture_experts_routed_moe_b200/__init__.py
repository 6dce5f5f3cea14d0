"""Routed mixture-of-experts expert forward for NVIDIA B200 (sm_100a).

Thin Python binding over the C ABI in ``include/moe_b200.h`` (library
``libmoe_b200.so``, built in-tree by ``_build.py``). Every step of the forward
runs in the library's CUDA kernels; this module only marshals arguments:
torch tensors provide device memory, ``torch.cuda.current_stream()`` the
stream. There is no CPU fallback: if the library is missing or cannot be
loaded, every entry point raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoe_b200.so")

MOE_OK = 0
STATUS = {
    0: "MOE_OK", -1: "MOE_ERR_INVALID_ARG", -2: "MOE_ERR_UNSUPPORTED", -3: "MOE_ERR_SCALE_FORMAT",
    -4: "MOE_ERR_WORKSPACE", -5: "MOE_ERR_CUDA", -6: "MOE_ERR_DEVICE_TIMEOUT", -7: "MOE_ERR_DEVICE_INDEX",
    -8: "MOE_ERR_SCRATCH_LIMIT",
}
WDTYPE = {"bf16": 0, "e4m3": 1, "e2m1": 2}
PATH = {"auto": 0, "prefill": 1, "decode": 2, "fused": 3}
ACT = {"silu": 0, "gelu": 1, "relu": 2}
PATH_NAMES = {v: k for k, v in PATH.items()}
EXPORTS = ["moe_route", "moe_workspace_size", "moe_forward", "moe_forward_timed", "moe_workspace_query",
           "moe_read_device_status", "moe_status_string", "moe_version", "moe_forward_noalloc",
           "moe_set_test_hooks", "moe_router", "moe_forward_noalloc_status"]


class MoeError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)} ({status_string(status)})")


class MoeShape(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("H", ctypes.c_int32), ("I", ctypes.c_int32), ("E", ctypes.c_int32),
                ("k", ctypes.c_int32), ("wdtype", ctypes.c_int32), ("path", ctypes.c_int32), ("act", ctypes.c_int32)]


class MoeWorkspaceLayout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in
                ("status", "hdr", "cnt", "mt_base", "row_src", "slot_row", "xa", "xs", "h", "hs", "y", "total")] + \
               [(n, ctypes.c_int32) for n in ("bm", "path", "m_rows", "reserved")]


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded CUDA library (raises if it is missing: there is no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing; build it with "
                              "`python -m mixture_experts_routed_moe_b200._build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
        L.moe_route.argtypes = [vp, i32, i32, i32, vp, vp, vp]
        L.moe_route.restype = i32
        L.moe_workspace_size.argtypes = [ctypes.POINTER(MoeShape)]
        L.moe_workspace_size.restype = sz
        fwd = [ctypes.POINTER(MoeShape), vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.moe_forward.argtypes = fwd
        L.moe_forward.restype = i32
        L.moe_forward_timed.argtypes = fwd + [ctypes.POINTER(vp), i32]
        L.moe_forward_timed.restype = i32
        L.moe_workspace_query.argtypes = [ctypes.POINTER(MoeShape), ctypes.POINTER(MoeWorkspaceLayout)]
        L.moe_workspace_query.restype = i32
        L.moe_read_device_status.argtypes = [vp, vp]
        L.moe_read_device_status.restype = i32
        L.moe_status_string.argtypes = [i32]
        L.moe_status_string.restype = ctypes.c_char_p
        L.moe_forward_noalloc.argtypes = [ctypes.POINTER(MoeShape), vp, vp, vp, vp, vp, vp, vp, vp, vp]
        L.moe_forward_noalloc.restype = i32
        L.moe_forward_noalloc_status.argtypes = [vp]
        L.moe_forward_noalloc_status.restype = i32
        L.moe_router.argtypes = [vp, vp, i32, i32, i32, i32, vp, vp, vp, vp]
        L.moe_router.restype = i32
        L.moe_set_test_hooks.argtypes = [i32, ctypes.c_uint64]
        L.moe_set_test_hooks.restype = i32
        L.moe_version.argtypes = []
        L.moe_version.restype = i32
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().moe_status_string(int(status)).decode()


def _check(status: int, what: str):
    if status != MOE_OK:
        raise MoeError(status, what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


_FLOAT8 = getattr(torch, "float8_e4m3fn", None)


def _need(t, name, dtypes, ndim, shape=None, cuda=True):
    """The library reads raw device pointers: check what it cannot (type,
    rank, sizes, contiguity, device) before handing one over. ``shape`` lists
    the expected sizes; ``cuda`` False leaves the device to a later check."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor, got {type(t).__name__}")
    if t.dtype not in dtypes:
        raise ValueError(f"{name}: dtype {t.dtype}, expected {' or '.join(str(d) for d in dtypes)}")
    if t.dim() != ndim:
        raise ValueError(f"{name}: {t.dim()}-D, expected {ndim}-D")
    if shape is not None and tuple(t.shape) != tuple(int(v) for v in shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(int(v) for v in shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if cuda and not t.is_cuda:
        raise ValueError(f"{name} must be on a CUDA device")


def _same_device(device, **tensors):
    """Every tensor on ``device`` (a CUDA device): the library launches on the
    current device and stream, so one tensor elsewhere would be read from the
    wrong GPU."""
    if device.type != "cuda":
        raise ValueError(f"x must be on a CUDA device, not {device}")
    for name, t in tensors.items():
        if t is not None and t.device != device:
            raise ValueError(f"{name} is on {t.device}, x on {device}: all tensors must share one CUDA device")


def _stream(stream=None, device=None):
    s = torch.cuda.current_stream(device) if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def make_shape(T, H, I, E, k, wdtype="bf16", path="auto", act="silu") -> MoeShape:
    return MoeShape(int(T), int(H), int(I), int(E), int(k), WDTYPE[wdtype] if isinstance(wdtype, str) else int(wdtype),
                    PATH[path] if isinstance(path, str) else int(path), ACT[act] if isinstance(act, str) else int(act))


def workspace_size(shape: MoeShape) -> int:
    n = lib().moe_workspace_size(ctypes.byref(shape))
    if n == 0:
        raise MoeError(-1, "moe_workspace_size")
    return int(n)


def workspace_layout(shape: MoeShape) -> MoeWorkspaceLayout:
    lay = MoeWorkspaceLayout()
    _check(lib().moe_workspace_query(ctypes.byref(shape), ctypes.byref(lay)), "moe_workspace_query")
    return lay


def alloc_workspace(shape: MoeShape, device=None) -> torch.Tensor:
    """A device buffer of moe_workspace_size(shape) bytes (torch allocates it)."""
    return torch.empty(workspace_size(shape), dtype=torch.uint8, device=device or "cuda")


def route(logits: torch.Tensor, k: int, topk_idx: torch.Tensor | None = None, topk_w: torch.Tensor | None = None,
          stream=None):
    """moe_route: fp32 logits [T,E] -> (int32 [T,k], fp32 [T,k])."""
    _need(logits, "logits", (torch.float32,), 2, cuda=False)
    T, E = logits.shape
    if topk_idx is None:
        topk_idx = torch.empty((T, k), dtype=torch.int32, device=logits.device)
    if topk_w is None:
        topk_w = torch.empty((T, k), dtype=torch.float32, device=logits.device)
    _need(topk_idx, "topk_idx", (torch.int32,), 2, (T, k), cuda=False)
    _need(topk_w, "topk_w", (torch.float32,), 2, (T, k), cuda=False)
    _same_device(logits.device, topk_idx=topk_idx, topk_w=topk_w)
    with torch.cuda.device(logits.device):
        _check(lib().moe_route(_ptr(logits), T, E, k, _ptr(topk_idx), _ptr(topk_w), _stream(stream, logits.device)),
               "moe_route")
    return topk_idx, topk_w


def _check_forward_args(x, topk_idx, topk_w, w_gate_up, w_down, sw_gate_up, sw_down, out, workspace=None):
    """Checks every tensor of a forward call against the layer the weights
    define (E experts, [gate; up] rows 2I, hidden H, top-k from topk_idx) and
    returns (T, H, I, E, k, wdtype). Sizes first, then that all share x's CUDA
    device: nothing reaches the library unless every pointer covers the
    extent the kernels will read or write."""
    _need(x, "x", (torch.bfloat16,), 2, cuda=False)
    T, H = x.shape
    _need(topk_idx, "topk_idx", (torch.int32,), 2, cuda=False)
    k = topk_idx.shape[1]
    _need(topk_idx, "topk_idx", (torch.int32,), 2, (T, k), cuda=False)
    _need(topk_w, "topk_w", (torch.float32,), 2, (T, k), cuda=False)
    # bf16 weights, e4m3 codes (float8_e4m3fn) or packed e2m1 codes (uint8, two per byte)
    wtypes = (torch.bfloat16, torch.uint8) + ((_FLOAT8,) if _FLOAT8 is not None else ())
    _need(w_gate_up, "w_gate_up", wtypes, 3, cuda=False)
    E, twoI = w_gate_up.shape[0], w_gate_up.shape[1]
    if twoI % 2 != 0:
        raise ValueError(f"w_gate_up: {twoI} rows per expert, expected 2*I (gate rows, then up rows)")
    I = twoI // 2
    fp8 = _FLOAT8 is not None and w_gate_up.dtype == _FLOAT8
    fp4 = w_gate_up.dtype == torch.uint8
    pk = 2 if fp4 else 1  # elements per stored byte or element along the reduction dimension
    _need(w_gate_up, "w_gate_up", wtypes, 3, (E, 2 * I, H // pk), cuda=False)
    _need(w_down, "w_down", (w_gate_up.dtype,), 3, (E, H, I // pk), cuda=False)
    if fp8 or fp4:
        # UE8M0 bytes: one per 128x128 block (e4m3) or per row and 32 elements (e2m1);
        # None makes the library refuse with MOE_ERR_SCALE_FORMAT
        g_gu, g_d = ((2 * I // 128, H // 128), (H // 128, I // 128)) if fp8 else ((2 * I, H // 32), (H, I // 32))
        if sw_gate_up is not None:
            _need(sw_gate_up, "sw_gate_up", (torch.uint8,), 3, (E,) + g_gu, cuda=False)
        if sw_down is not None:
            _need(sw_down, "sw_down", (torch.uint8,), 3, (E,) + g_d, cuda=False)
    elif sw_gate_up is not None or sw_down is not None:
        raise ValueError("block scales were given for bf16 experts")
    if out is not None:
        _need(out, "out", (torch.bfloat16,), 2, (T, H), cuda=False)
    if workspace is not None:
        _need(workspace, "workspace", (torch.uint8,), 1, cuda=False)
    _same_device(x.device, topk_idx=topk_idx, topk_w=topk_w, w_gate_up=w_gate_up, w_down=w_down,
                 sw_gate_up=sw_gate_up, sw_down=sw_down, out=out, workspace=workspace)
    return T, H, I, E, k, ("e4m3" if fp8 else "e2m1" if fp4 else "bf16")


def forward(x, topk_idx, topk_w, w_gate_up, w_down, sw_gate_up=None, sw_down=None, out=None, workspace=None,
            path="auto", stream=None, events=None, act="silu"):
    """moe_forward: bf16 x [T,H] with routing [T,k] through experts
    w_gate_up [E,2I,H], w_down [E,H,I] (bf16, or float8_e4m3fn with uint8 UE8M0
    block scales) -> bf16 out [T,H]; act is the gate activation ("silu" for
    SwiGLU, "gelu" for GeGLU, "relu" for ReGLU). Returns (out, workspace)."""
    T, H, I, E, k, wdtype = _check_forward_args(x, topk_idx, topk_w, w_gate_up, w_down, sw_gate_up, sw_down, out,
                                                workspace)
    shape = make_shape(T, H, I, E, k, wdtype, path, act)
    with torch.cuda.device(x.device):
        if out is None:
            out = torch.empty((T, H), dtype=torch.bfloat16, device=x.device)
        if workspace is None:
            workspace = alloc_workspace(shape, x.device)
        st = stream or torch.cuda.current_stream(x.device)
        args = [ctypes.byref(shape), _ptr(x), _ptr(topk_idx), _ptr(topk_w), _ptr(w_gate_up), _ptr(w_down),
                _ptr(sw_gate_up), _ptr(sw_down), _ptr(out), _ptr(workspace), workspace.numel(), _stream(st)]
        if events is None:
            _check(lib().moe_forward(*args), "moe_forward")
        else:
            for e in events:  # torch creates the CUDA event lazily, on its first record
                if not e.cuda_event:
                    e.record(st)
            ev = (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events])
            _check(lib().moe_forward_timed(*args, ev, len(events)), "moe_forward_timed")
    return out, workspace


def forward_noalloc(x, topk_idx, topk_w, w_gate_up, w_down, sw_gate_up=None, sw_down=None, out=None, path="auto",
                    stream=None, act="silu"):
    """moe_forward_noalloc: the forward with the library's own fixed scratch
    array instead of a caller workspace, for callers that cannot allocate device
    memory (only ``out`` is allocated here when not given). Calls share the
    array, so calls whose GPU work overlaps must be ordered by the caller."""
    T, H, I, E, k, wdtype = _check_forward_args(x, topk_idx, topk_w, w_gate_up, w_down, sw_gate_up, sw_down, out)
    shape = make_shape(T, H, I, E, k, wdtype, path, act)
    with torch.cuda.device(x.device):
        if out is None:
            out = torch.empty((T, H), dtype=torch.bfloat16, device=x.device)
        _check(lib().moe_forward_noalloc(ctypes.byref(shape), _ptr(x), _ptr(topk_idx), _ptr(topk_w),
                                         _ptr(w_gate_up), _ptr(w_down), _ptr(sw_gate_up), _ptr(sw_down), _ptr(out),
                                         _stream(stream, x.device)),
               "moe_forward_noalloc")
    return out


def noalloc_device_status(device=None, stream=None) -> int:
    """Synchronises the stream and returns the device status of the last
    forward_noalloc on `device` (read from the library's own scratch)."""
    device = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    with torch.cuda.device(device):
        return int(lib().moe_forward_noalloc_status(_stream(stream, device)))


def read_device_status(workspace: torch.Tensor, stream=None) -> int:
    """Synchronises the stream and returns the device status of the last forward on `workspace`."""
    with torch.cuda.device(workspace.device):
        return int(lib().moe_read_device_status(_ptr(workspace), _stream(stream, workspace.device)))


def router(x: torch.Tensor, w_router: torch.Tensor, k: int, logits: bool = False, stream=None):
    """moe_router: logits = x w_router^T (bf16 in, fp32 accumulate) and the
    top-k routing on them, in one kernel. x bf16 [T,H], w_router bf16 [E,H].
    Returns (topk_idx int32 [T,k], topk_w fp32 [T,k]) and, with logits=True,
    the fp32 logits [T,E] as a third element."""
    _need(x, "x", (torch.bfloat16,), 2, cuda=False)
    T, H = x.shape
    _need(w_router, "w_router", (torch.bfloat16,), 2, cuda=False)
    E = w_router.shape[0]
    _need(w_router, "w_router", (torch.bfloat16,), 2, (E, H), cuda=False)
    _same_device(x.device, w_router=w_router)
    with torch.cuda.device(x.device):
        idx = torch.empty((T, k), dtype=torch.int32, device=x.device)
        w = torch.empty((T, k), dtype=torch.float32, device=x.device)
        lg = torch.empty((T, E), dtype=torch.float32, device=x.device) if logits else None
        _check(lib().moe_router(_ptr(x), _ptr(w_router), T, H, E, k, _ptr(lg), _ptr(idx), _ptr(w),
                                _stream(stream, x.device)),
               "moe_router")
    return (idx, w, lg) if logits else (idx, w)


def set_test_hooks(stall_gate_up_loads: bool = False, wait_limit_ns: int = 0) -> None:
    """Failure-detection test switches (moe_set_test_hooks): the limit of every
    bounded device wait (0 = the 2 s default) and a stall of the prefill
    gate/up GEMM's loads. Raises MoeError on values out of range."""
    _check(lib().moe_set_test_hooks(int(bool(stall_gate_up_loads)), int(wait_limit_ns)), "moe_set_test_hooks")


class MoELayer:
    """A routed MoE layer whose expert weights live on the GPU: ``layer(x, logits)``
    runs moe_route then moe_forward and returns bf16 [T,H]. The workspace is
    allocated once per shape and reused."""

    def __init__(self, w_gate_up, w_down, k, sw_gate_up=None, sw_down=None, path="auto", act="silu"):
        self.w_gate_up, self.w_down = w_gate_up, w_down
        self.sw_gate_up, self.sw_down = sw_gate_up, sw_down
        self.k, self.path, self.act = int(k), path, act
        self.E, twoI = w_gate_up.shape[0], w_gate_up.shape[1]
        self.H = w_down.shape[1]
        self.I = twoI // 2
        self._ws = {}

    def _workspace(self, T, device):
        wdtype = {torch.float8_e4m3fn: "e4m3", torch.uint8: "e2m1"}.get(self.w_gate_up.dtype, "bf16")
        shape = make_shape(T, self.H, self.I, self.E, self.k, wdtype, self.path, self.act)
        key = (T, str(device))
        if key not in self._ws:
            self._ws[key] = alloc_workspace(shape, device)
        return self._ws[key]

    def __call__(self, x, logits, out=None, events=None):
        idx, w = route(logits, self.k)
        out, _ = forward(x, idx, w, self.w_gate_up, self.w_down, self.sw_gate_up, self.sw_down, out=out,
                         workspace=self._workspace(x.shape[0], x.device), path=self.path, events=events,
                         act=self.act)
        return out


class MoEGraph:
    """One layer step (moe_route + moe_forward) captured once in a CUDA graph for
    a fixed token count, on static device buffers ``x``, ``logits`` and ``out``.
    ``replay()`` reruns the captured kernels with no host-side work per step;
    ``__call__(x, logits)`` copies new inputs into the static buffers first.
    The library's launches are capture-safe: no allocation, no host
    synchronisation, and one-time set-up done by the eager warm-up call."""

    def __init__(self, layer: "MoELayer", T: int, device=None):
        device = torch.device(device or "cuda")
        self.layer = layer
        self.x = torch.zeros((T, layer.H), dtype=torch.bfloat16, device=device)
        self.logits = torch.zeros((T, layer.E), dtype=torch.float32, device=device)
        self.out = torch.empty((T, layer.H), dtype=torch.bfloat16, device=device)
        side = torch.cuda.Stream(device=device)
        side.wait_stream(torch.cuda.current_stream(device))
        with torch.cuda.stream(side):  # eager warm-up: workspace, kernel set-up
            layer(self.x, self.logits, out=self.out)
        torch.cuda.current_stream(device).wait_stream(side)
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            layer(self.x, self.logits, out=self.out)

    def replay(self) -> torch.Tensor:
        self.graph.replay()
        return self.out

    def __call__(self, x=None, logits=None) -> torch.Tensor:
        if x is not None:
            self.x.copy_(x, non_blocking=True)
        if logits is not None:
            self.logits.copy_(logits, non_blocking=True)
        return self.replay()


class MoEPipeline:
    """Layer steps from host memory to host memory for a stream of batches,
    with the copies overlapped with the compute: batch i's x and logits are
    copied in on one stream while batch i-1 runs, and batch i-1's output is
    copied out on another while batch i runs. ``depth`` MoEGraph instances
    (static device buffers and a captured graph each) take the batches in
    turn; their graphs run in submission order on one compute stream, so they
    share the layer's workspace. Events keep a buffer set from being refilled
    before its graph has read it and its output from being overwritten before
    it was copied out. Host tensors must be pinned for the copies to overlap;
    a caller reads ``out_host`` of a batch after ``done(i)`` or ``synchronize()``."""

    def __init__(self, layer: "MoELayer", T: int, device=None, depth: int = 2):
        if depth < 2:
            raise ValueError("depth must be at least 2 for the copies to overlap the compute")
        device = torch.device(device or "cuda")
        self.device = device
        self.depth = depth
        self.graphs = [MoEGraph(layer, T, device) for _ in range(depth)]
        self.copy_in = torch.cuda.Stream(device=device)
        self.compute = torch.cuda.Stream(device=device)
        self.copy_out = torch.cuda.Stream(device=device)
        self.inputs_ready = [torch.cuda.Event() for _ in range(depth)]
        self.computed = [torch.cuda.Event() for _ in range(depth)]
        self.output_read = [torch.cuda.Event() for _ in range(depth)]
        self.n = 0

    def submit(self, x_host: torch.Tensor, logits_host: torch.Tensor, out_host: torch.Tensor, before_compute=None):
        """Queue one batch; returns its sequence number. ``before_compute``, if
        given, is called with the compute stream current just before the
        batch's graph (for work that must run in the compute order)."""
        s = self.n % self.depth
        g = self.graphs[s]
        reuse = self.n >= self.depth
        with torch.cuda.stream(self.copy_in):
            if reuse:
                self.copy_in.wait_event(self.computed[s])  # the slot's previous graph has read its inputs
            g.x.copy_(x_host, non_blocking=True)
            g.logits.copy_(logits_host, non_blocking=True)
            self.inputs_ready[s].record(self.copy_in)
        with torch.cuda.stream(self.compute):
            self.compute.wait_event(self.inputs_ready[s])
            if reuse:
                self.compute.wait_event(self.output_read[s])  # the slot's previous output was copied out
            if before_compute is not None:
                before_compute()
            g.graph.replay()
            self.computed[s].record(self.compute)
        with torch.cuda.stream(self.copy_out):
            self.copy_out.wait_event(self.computed[s])
            out_host.copy_(g.out, non_blocking=True)
            self.output_read[s].record(self.copy_out)
        self.n += 1
        return self.n - 1

    def done(self, i: int) -> bool:
        """True once batch i's output has been copied out (only the last
        ``depth`` batches can be asked)."""
        if not (self.n - self.depth <= i < self.n):
            raise ValueError("only the last depth batches can be queried")
        return self.output_read[i % self.depth].query()

    def synchronize(self):
        for st in (self.copy_in, self.compute, self.copy_out):
            st.synchronize()


__all__ = ["lib", "route", "forward", "forward_noalloc", "noalloc_device_status", "MoEGraph", "MoEPipeline", "workspace_size", "workspace_layout", "alloc_workspace",
           "read_device_status", "set_test_hooks", "router", "make_shape", "MoELayer", "MoeError", "MoeShape", "EXPORTS", "STATUS",
           "status_string", "PATH", "WDTYPE", "ACT"]
