"""Thin ctypes binding of libmoe.so (C ABI in include/moe.h).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels. torch supplies device memory and the current stream. If the library
is missing or cannot be loaded the first call raises; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

from .workloads import BF16, E2M1, E4M3, F32, Spec

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoe.so")

MOE_F32, MOE_BF16, MOE_E4M3, MOE_E2M1 = 0, 1, 2, 3
_DT = {F32: MOE_F32, BF16: MOE_BF16, E4M3: MOE_E4M3, E2M1: MOE_E2M1}
_TORCH = {F32: torch.float32, BF16: torch.bfloat16, E4M3: torch.uint8}

STATUS = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED", 3: "MOE_ERR_CUDA",
          4: "MOE_ERR_CAPACITY", 5: "MOE_ERR_TIMEOUT", 6: "MOE_ERR_NONFINITE"}

EXPORTS = ("moe_workspace_bytes", "moe_workspace_init", "moe_route", "moe_dispatch",
           "moe_grouped_ffn", "moe_combine", "moe_layer", "moe_layer_bufs", "moe_layer_workspace_bytes",
           "moe_poll_status", "moe_status_string", "moe_dispatch_noalloc", "moe_pack_mx_scales",
           "moe_layer_overlap", "moe_ep_sizes", "moe_ep_workspace_init", "moe_ep_count", "moe_ep_layout",
           "moe_ep_dispatch", "moe_ep_grouped_ffn", "moe_ep_combine")


class MoeError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn}: {STATUS.get(code, code)}")
        self.code = code


class moe_shape(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("H", ctypes.c_int64), ("E", ctypes.c_int64),
                ("topk", ctypes.c_int64), ("I", ctypes.c_int64),
                ("act_dtype", ctypes.c_int32), ("xq_dtype", ctypes.c_int32),
                ("weight_dtype", ctypes.c_int32), ("h_dtype", ctypes.c_int32),
                ("y_dtype", ctypes.c_int32), ("out_dtype", ctypes.c_int32),
                ("renorm", ctypes.c_int32), ("identity_experts", ctypes.c_int32),
                ("cap_rows", ctypes.c_int64), ("quant_block", ctypes.c_int32),
                ("flags", ctypes.c_int32)]


class moe_dispatch_bufs(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("xq", "xs", "counts", "offsets", "row_src", "pos", "hq", "hs")]


class moe_weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("w_gate", "w_up", "w_down", "s_gate", "s_up", "s_down")]


class moe_overlap(ctypes.Structure):
    _fields_ = [("dispatch_stream", ctypes.c_void_p), ("fork_event", ctypes.c_void_p),
                ("join_event", ctypes.c_void_p), ("dispatch_sms", ctypes.c_int32),
                ("ffn_sms", ctypes.c_int32)]


MOE_EP_SENTINEL, MOE_EP_FENCE = 0, 1


class moe_ep(ctypes.Structure):
    _fields_ = [("ranks", ctypes.c_int32), ("rank", ctypes.c_int32), ("protocol", ctypes.c_int32),
                ("reserved", ctypes.c_int32), ("t_max", ctypes.c_int64)]


class moe_ep_windows(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("xq", "xs", "row_src", "hq", "hs", "y", "ws")]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libmoe.so (raises if it is absent: build it with
    ``python -m combine_softmax_top_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing; build it with "
                               "`python -m combine_softmax_top_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, S = ctypes.c_void_p, ctypes.POINTER(moe_shape)
        sig = {
            "moe_workspace_bytes": [S, ctypes.POINTER(ctypes.c_size_t)],
            "moe_workspace_init": [S, P, ctypes.c_size_t, P],
            "moe_route": [S, P, P, P, P, P],
            "moe_dispatch": [S, P, P, P, ctypes.POINTER(moe_dispatch_bufs), P],
            "moe_grouped_ffn": [S, ctypes.POINTER(moe_dispatch_bufs), ctypes.POINTER(moe_weights),
                                P, P, P],
            "moe_combine": [S, ctypes.POINTER(moe_dispatch_bufs), P, P, P, P, P],
            "moe_layer": [S, P, P, ctypes.POINTER(moe_weights), P, P, P],
            "moe_layer_bufs": [S, P, P, ctypes.POINTER(moe_weights), P, P,
                               ctypes.POINTER(moe_dispatch_bufs), P, P, P, P],
            "moe_layer_workspace_bytes": [S, ctypes.POINTER(ctypes.c_size_t)],
            "moe_poll_status": [P, P],
            "moe_dispatch_noalloc": [S, P, P, ctypes.POINTER(moe_dispatch_bufs), P],
            "moe_status_string": [ctypes.c_int],
            "moe_pack_mx_scales": [ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, P, P, P],
            "moe_layer_overlap": [S, P, P, ctypes.POINTER(moe_weights), P, P, P,
                                  ctypes.POINTER(moe_overlap)],
            "moe_ep_sizes": [S, ctypes.POINTER(moe_ep), ctypes.POINTER(ctypes.c_int64),
                             ctypes.POINTER(ctypes.c_size_t)],
            "moe_ep_workspace_init": [S, ctypes.POINTER(moe_ep), ctypes.POINTER(moe_ep_windows), P],
            "moe_ep_count": [S, ctypes.POINTER(moe_ep), P, ctypes.POINTER(moe_ep_windows), P],
            "moe_ep_layout": [S, ctypes.POINTER(moe_ep), ctypes.POINTER(moe_ep_windows), P],
            "moe_ep_dispatch": [S, ctypes.POINTER(moe_ep), P, P, ctypes.POINTER(moe_ep_windows), P, P],
            "moe_ep_grouped_ffn": [S, ctypes.POINTER(moe_ep), ctypes.POINTER(moe_weights),
                                   ctypes.POINTER(moe_ep_windows), P],
            "moe_ep_combine": [S, ctypes.POINTER(moe_ep), P, P, ctypes.POINTER(moe_ep_windows), P, P],
        }
        for name, args in sig.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = ctypes.c_char_p if name == "moe_status_string" else ctypes.c_int
        _lib = L
    return _lib


def _ptr(t) -> ctypes.c_void_p:
    if t is None:
        return ctypes.c_void_p(0)
    if isinstance(t, int):
        return ctypes.c_void_p(t)
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(fn: str, rc: int) -> None:
    if rc != 0:
        raise MoeError(fn, rc)


def make_shape(s: Spec, T: int | None = None) -> moe_shape:
    sh = moe_shape()
    sh.T = s.T if T is None else T
    sh.H, sh.E, sh.topk, sh.I = s.H, s.E, s.k, s.I
    sh.act_dtype, sh.xq_dtype = _DT[s.act], _DT[s.xq]
    sh.weight_dtype, sh.h_dtype, sh.y_dtype, sh.out_dtype = _DT[s.weight], _DT[s.h], _DT[s.y], _DT[s.out]
    sh.renorm, sh.identity_experts = s.renorm, s.identity
    sh.cap_rows = s.cap_rows
    # MOE_FLAG_SHARED_EXPERT = 1, MOE_FLAG_COMPACT = 2
    sh.quant_block, sh.flags = 128, (1 if s.shared else 0) | (2 if s.compact else 0)
    return sh


# ------------------------------------------------------------ raw C calls --

def moe_workspace_bytes(shape: moe_shape) -> int:
    n = ctypes.c_size_t(0)
    _check("moe_workspace_bytes", lib().moe_workspace_bytes(ctypes.byref(shape), ctypes.byref(n)))
    return n.value


def moe_workspace_init(shape: moe_shape, ws: torch.Tensor, stream=None) -> None:
    _check("moe_workspace_init", lib().moe_workspace_init(ctypes.byref(shape), _ptr(ws),
                                                         ws.numel() * ws.element_size(), _stream(stream)))


def moe_route(shape, logits, topk_idx, topk_w, ws, stream=None) -> None:
    _check("moe_route", lib().moe_route(ctypes.byref(shape), _ptr(logits), _ptr(topk_idx),
                                        _ptr(topk_w), _ptr(ws), _stream(stream)))


def moe_dispatch(shape, x, topk_idx, ws, bufs: moe_dispatch_bufs, stream=None) -> None:
    _check("moe_dispatch", lib().moe_dispatch(ctypes.byref(shape), _ptr(x), _ptr(topk_idx),
                                              _ptr(ws), ctypes.byref(bufs), _stream(stream)))


def moe_grouped_ffn(shape, bufs: moe_dispatch_bufs, w: moe_weights, ws, y, stream=None) -> None:
    _check("moe_grouped_ffn", lib().moe_grouped_ffn(ctypes.byref(shape), ctypes.byref(bufs),
                                                    ctypes.byref(w), _ptr(ws), _ptr(y),
                                                    _stream(stream)))


def moe_combine(shape, bufs: moe_dispatch_bufs, y, topk_w, ws, out, stream=None) -> None:
    _check("moe_combine", lib().moe_combine(ctypes.byref(shape), ctypes.byref(bufs), _ptr(y),
                                            _ptr(topk_w), _ptr(ws), _ptr(out), _stream(stream)))


def moe_layer_workspace_bytes(shape: moe_shape) -> int:
    n = ctypes.c_size_t(0)
    _check("moe_layer_workspace_bytes",
           lib().moe_layer_workspace_bytes(ctypes.byref(shape), ctypes.byref(n)))
    return n.value


def moe_layer(shape, x, logits, w: moe_weights, ws, out, stream=None) -> None:
    """The whole layer with every intermediate inside `ws` (of at least
    moe_layer_workspace_bytes bytes)."""
    _check("moe_layer", lib().moe_layer(ctypes.byref(shape), _ptr(x), _ptr(logits),
                                        ctypes.byref(w), _ptr(ws), _ptr(out), _stream(stream)))


def moe_layer_bufs(shape, x, logits, w: moe_weights, topk_idx, topk_w, bufs: moe_dispatch_bufs, y, ws,
                   out, stream=None) -> None:
    _check("moe_layer_bufs", lib().moe_layer_bufs(ctypes.byref(shape), _ptr(x), _ptr(logits),
                                                  ctypes.byref(w), _ptr(topk_idx), _ptr(topk_w),
                                                  ctypes.byref(bufs), _ptr(y), _ptr(ws), _ptr(out),
                                                  _stream(stream)))


def moe_layer_overlap(shape, x, logits, w: moe_weights, ws, out, ov: moe_overlap, stream=None) -> None:
    """moe_layer with dispatch on ov.dispatch_stream beside the grouped FFN."""
    _check("moe_layer_overlap", lib().moe_layer_overlap(ctypes.byref(shape), _ptr(x), _ptr(logits),
                                                        ctypes.byref(w), _ptr(ws), _ptr(out), _stream(stream),
                                                        ctypes.byref(ov)))


def moe_ep_sizes(shape, ep: moe_ep) -> tuple[int, int]:
    """(rows of one rank's windows, bytes of one rank's workspace)."""
    rows, nb = ctypes.c_int64(0), ctypes.c_size_t(0)
    _check("moe_ep_sizes", lib().moe_ep_sizes(ctypes.byref(shape), ctypes.byref(ep), ctypes.byref(rows),
                                              ctypes.byref(nb)))
    return rows.value, nb.value


def moe_ep_workspace_init(shape, ep: moe_ep, win: moe_ep_windows, stream=None) -> None:
    _check("moe_ep_workspace_init", lib().moe_ep_workspace_init(ctypes.byref(shape), ctypes.byref(ep),
                                                                ctypes.byref(win), _stream(stream)))


def moe_ep_count(shape, ep: moe_ep, topk_idx, win: moe_ep_windows, stream=None) -> None:
    _check("moe_ep_count", lib().moe_ep_count(ctypes.byref(shape), ctypes.byref(ep), _ptr(topk_idx),
                                              ctypes.byref(win), _stream(stream)))


def moe_ep_layout(shape, ep: moe_ep, win: moe_ep_windows, stream=None) -> None:
    _check("moe_ep_layout", lib().moe_ep_layout(ctypes.byref(shape), ctypes.byref(ep), ctypes.byref(win),
                                                _stream(stream)))


def moe_ep_dispatch(shape, ep: moe_ep, x, topk_idx, win: moe_ep_windows, pos, stream=None) -> None:
    _check("moe_ep_dispatch", lib().moe_ep_dispatch(ctypes.byref(shape), ctypes.byref(ep), _ptr(x),
                                                    _ptr(topk_idx), ctypes.byref(win), _ptr(pos),
                                                    _stream(stream)))


def moe_ep_grouped_ffn(shape, ep: moe_ep, w: moe_weights, win: moe_ep_windows, stream=None) -> None:
    _check("moe_ep_grouped_ffn", lib().moe_ep_grouped_ffn(ctypes.byref(shape), ctypes.byref(ep), ctypes.byref(w),
                                                          ctypes.byref(win), _stream(stream)))


def moe_ep_combine(shape, ep: moe_ep, pos, topk_w, win: moe_ep_windows, out, stream=None) -> None:
    _check("moe_ep_combine", lib().moe_ep_combine(ctypes.byref(shape), ctypes.byref(ep), _ptr(pos), _ptr(topk_w),
                                                  ctypes.byref(win), _ptr(out), _stream(stream)))


def moe_pack_mx_scales(src: torch.Tensor, stream=None) -> torch.Tensor:
    """MX FP4 weight scales [n, rows, cols/32] (uint8, device) -> the scale
    atoms [n, rows/128, cols/128, 512] moe_weights wants (moe_pack_mx_scales)."""
    n, rows, groups = src.shape
    src = src.contiguous()
    dst = torch.empty((n, rows // 128, groups * 32 // 128, 512), dtype=torch.uint8, device=src.device)
    _check("moe_pack_mx_scales", lib().moe_pack_mx_scales(n, rows, groups * 32, _ptr(src), _ptr(dst),
                                                           _stream(stream)))
    return dst


def moe_dispatch_noalloc(shape, x, topk_idx, bufs: moe_dispatch_bufs, stream=None) -> None:
    """moe_dispatch for callers that cannot supply a workspace (the library's
    fixed device array is used instead; see include/moe.h)."""
    _check("moe_dispatch_noalloc", lib().moe_dispatch_noalloc(ctypes.byref(shape), _ptr(x),
                                                              _ptr(topk_idx), ctypes.byref(bufs),
                                                              _stream(stream)))


def moe_poll_status(ws, stream=None) -> int:
    return int(lib().moe_poll_status(_ptr(ws), _stream(stream)))


def moe_status_string(code: int) -> str:
    return lib().moe_status_string(int(code)).decode()


# ------------------------------------------------------------ convenience --

@dataclass
class Buffers:
    """Device buffers of one layer (torch tensors; marshalling helpers only)."""
    shape: moe_shape
    spec: Spec
    ws: torch.Tensor
    topk_idx: torch.Tensor
    topk_w: torch.Tensor
    xq: torch.Tensor
    xs: torch.Tensor | None
    counts: torch.Tensor
    offsets: torch.Tensor
    row_src: torch.Tensor
    pos: torch.Tensor
    hq: torch.Tensor | None
    hs: torch.Tensor | None
    y: torch.Tensor | None
    out: torch.Tensor

    def dispatch_bufs(self) -> moe_dispatch_bufs:
        b = moe_dispatch_bufs()
        b.xq, b.xs = self.xq.data_ptr(), (self.xs.data_ptr() if self.xs is not None else 0)
        b.counts, b.offsets = self.counts.data_ptr(), self.offsets.data_ptr()
        b.row_src, b.pos = self.row_src.data_ptr(), self.pos.data_ptr()
        b.hq = self.hq.data_ptr() if self.hq is not None else 0
        b.hs = self.hs.data_ptr() if self.hs is not None else 0
        return b


def alloc_buffers(s: Spec, device="cuda", T: int | None = None, stream=None) -> Buffers:
    """Allocate every buffer the layer writes (through torch) and initialise
    the workspace."""
    sh = make_shape(s, T)
    T = sh.T
    ne, ks = s.E + s.shared, s.k + s.shared   # a shared expert adds one expert and one slot
    rows = s.rows(T)
    nws = moe_workspace_bytes(sh)
    ws = torch.empty(nws, dtype=torch.uint8, device=device)
    z = dict(device=device)
    bufs = Buffers(
        shape=sh, spec=s, ws=ws,
        topk_idx=torch.empty((T, ks), dtype=torch.int32, **z),
        topk_w=torch.empty((T, ks), dtype=torch.float32, **z),
        xq=torch.empty((rows, s.H), dtype=_TORCH[s.xq], **z),
        xs=torch.empty((rows, s.H // 128), dtype=torch.float32, **z) if s.xq == E4M3 else None,
        counts=torch.empty(ne, dtype=torch.int32, **z),
        offsets=torch.empty(ne, dtype=torch.int32, **z),
        row_src=torch.full((rows,), -1, dtype=torch.int32, **z),
        pos=torch.empty(T * ks, dtype=torch.int32, **z),
        hq=None if s.identity else torch.empty((rows, s.I), dtype=_TORCH[s.h], **z),
        hs=torch.empty((rows, s.I // 128), dtype=torch.float32, **z)
        if (not s.identity and s.h == E4M3) else None,
        y=None if s.identity else torch.empty((rows, s.H), dtype=_TORCH[s.y], **z),
        out=torch.empty((T, s.H), dtype=_TORCH[s.out], **z),
    )
    moe_workspace_init(sh, ws, stream)
    return bufs


def weights_struct(inp: dict) -> moe_weights:
    w = moe_weights()
    w.w_gate, w.w_up, w.w_down = (inp["w_gate"].data_ptr(), inp["w_up"].data_ptr(),
                                  inp["w_down"].data_ptr())
    for k in ("s_gate", "s_up", "s_down"):
        t = inp.get(k)
        setattr(w, k, t.data_ptr() if t is not None else 0)
    return w


def run_layer(b: Buffers, inp: dict, stream=None) -> None:
    """Enqueue one whole layer into `b`'s buffers (moe_layer_bufs) on the
    current stream."""
    w = weights_struct(inp) if not b.spec.identity else moe_weights()
    moe_layer_bufs(b.shape, inp["x"], inp["logits"], w, b.topk_idx, b.topk_w, b.dispatch_bufs(), b.y,
                   b.ws, b.out, stream)


@dataclass
class LayerWorkspace:
    """A workspace holding every intermediate of moe_layer, and the output."""
    shape: moe_shape
    spec: Spec
    ws: torch.Tensor
    out: torch.Tensor


def alloc_layer(s: Spec, device="cuda", stream=None) -> LayerWorkspace:
    sh = make_shape(s)
    ws = torch.empty(moe_layer_workspace_bytes(sh), dtype=torch.uint8, device=device)
    moe_workspace_init(sh, ws, stream)
    return LayerWorkspace(sh, s, ws, torch.empty((s.T, s.H), dtype=_TORCH[s.out], device=device))


def run_layer_ws(lw: LayerWorkspace, inp: dict, stream=None) -> None:
    """Enqueue one whole layer (moe_layer, intermediates in the workspace)."""
    w = weights_struct(inp) if not lw.spec.identity else moe_weights()
    moe_layer(lw.shape, inp["x"], inp["logits"], w, lw.ws, lw.out, stream)


class GreenPartition:
    """Two green contexts over disjoint SM sets of one device, one stream
    each: `dispatch_sms` SMs (rounded up by the driver to its split
    granularity) for dispatch, every other SM for the rest of the layer.
    Both sides must be confined: a kernel on an ordinary stream may run on
    any SM, so a persistent grouped FFN there can take the SMs of a
    dispatch-only green context and leave dispatch none, and the FFN's
    tile waits then run out. Made with the driver's SM-resource split
    (cuda.bindings); released by close()."""

    def __init__(self, dispatch_sms: int, index: int):
        from cuda.bindings import driver as cu
        self._cu = cu
        self._ctxs, self._streams = [], []

        def call(fn, *args):
            r = fn(*args)
            if r[0] != cu.CUresult.CUDA_SUCCESS:
                raise RuntimeError(f"{fn.__name__} failed: {r[0]}")
            return r[1] if len(r) == 2 else r[1:]

        try:
            call(cu.cuInit, 0)
            dev = call(cu.cuDeviceGet, index)
            sm = call(cu.cuDeviceGetDevResource, dev, cu.CUdevResourceType.CU_DEV_RESOURCE_TYPE_SM)
            groups, n, rest = call(cu.cuDevSmResourceSplitByCount, 1, sm, 0, int(dispatch_sms))
            if n < 1 or groups[0].sm.smCount < 1 or rest.sm.smCount < 1:
                raise RuntimeError(f"no SM split of {dispatch_sms} on device {index}")
            # dispatch: high priority, it is the producer the grouped FFN waits on
            for res, prio in ((groups[0], -1), (rest, 0)):
                desc = call(cu.cuDevResourceGenerateDesc, [res], 1)
                g = call(cu.cuGreenCtxCreate, desc, dev, cu.CUgreenCtxCreate_flags.CU_GREEN_CTX_DEFAULT_STREAM)
                self._ctxs.append(g)
                self._streams.append(call(cu.cuGreenCtxStreamCreate, g, cu.CUstream_flags.CU_STREAM_NON_BLOCKING,
                                          prio))
        except Exception:
            self.close()
            raise
        self.dispatch_sms = int(groups[0].sm.smCount)
        self.main_sms = int(rest.sm.smCount)
        self.dispatch_stream = int(self._streams[0])
        self.main_stream = int(self._streams[1])

    def close(self) -> None:
        cu = self._cu
        for st in self._streams:
            cu.cuStreamSynchronize(st)
            cu.cuStreamDestroy(st)
        for g in self._ctxs:
            cu.cuGreenCtxDestroy(g)
        self._streams, self._ctxs = [], []


class Overlap:
    """A dispatch stream and the fork/join events moe_layer_overlap orders it
    with (torch objects; the library only borrows their handles). Without
    green, the grouped FFN's persistent grid leaves dispatch_sms SMs free and
    dispatch runs on a second stream of the caller's context. With
    green=True the device enforces the split: dispatch runs on a green
    context of dispatch_sms SMs and the layer itself (route, counting pass,
    grouped FFN, combine) on a green context of all the other SMs
    (GreenPartition); `main` is that stream, and overlap_layer orders it
    after and before the caller's stream."""

    def __init__(self, dispatch_sms: int, ffn_sms: int = 0, green: bool = False, device=None):
        self.partition = None
        self.main = None
        if device is None:
            index = torch.cuda.current_device()
        elif isinstance(device, int):
            index = device
        else:
            index = torch.device(device).index or 0
        if green:
            self.partition = GreenPartition(dispatch_sms, index)
            self.stream = torch.cuda.ExternalStream(self.partition.dispatch_stream, device=index)
            self.main = torch.cuda.ExternalStream(self.partition.main_stream, device=index)
            dispatch_sms = self.partition.dispatch_sms
            ffn_sms = min(ffn_sms, self.partition.main_sms) if ffn_sms else self.partition.main_sms
        else:
            # a high-priority stream: dispatch is the producer the FFN waits on
            # (and high-priority streams never double as graph-capture streams)
            self.stream = torch.cuda.Stream(device=index, priority=-1)
        self.fork = torch.cuda.Event()
        self.join = torch.cuda.Event()
        # events exist once recorded: record both so their handles are real
        self.fork.record(self.stream)
        self.join.record(self.stream)
        torch.cuda.synchronize(index)
        self.ov = moe_overlap()
        self.ov.dispatch_stream = self.stream.cuda_stream
        self.ov.fork_event = self.fork.cuda_event
        self.ov.join_event = self.join.cuda_event
        self.ov.dispatch_sms = dispatch_sms
        self.ov.ffn_sms = ffn_sms

    def close(self) -> None:
        if self.partition is not None:
            torch.cuda.synchronize()
            self.partition.close()
            self.partition = None


def overlap_layer(shape, x, logits, w: moe_weights, ws, out, ov: Overlap, stream=None) -> None:
    """moe_layer_overlap on `stream`, or, for a green split, on its main
    stream ordered after the caller's stream and before whatever the caller
    enqueues next."""
    if ov.main is None:
        moe_layer_overlap(shape, x, logits, w, ws, out, ov.ov, stream)
        return
    cur = torch.cuda.current_stream() if stream is None else stream
    ov.main.wait_stream(cur)
    moe_layer_overlap(shape, x, logits, w, ws, out, ov.ov, ov.main)
    cur.wait_stream(ov.main)


def run_layer_overlap(lw: "LayerWorkspace", inp: dict, ov: Overlap, stream=None) -> None:
    """Enqueue one whole layer with dispatch beside the grouped FFN."""
    overlap_layer(lw.shape, inp["x"], inp["logits"], weights_struct(inp), lw.ws, lw.out, ov, stream)


# kernels the library launches per stage (mirrors the launch plan in csrc/)
_FFN_KERNELS = {F32: 2, BF16: 1, E4M3: 1, E2M1: 1}


def kernels_per_layer(s: Spec) -> int:
    """route + dispatch (+ its counting pass with compact windows) + grouped
    FFN + combine launches of one moe_layer."""
    return 3 + (1 if s.compact else 0) + (0 if s.identity else _FFN_KERNELS[s.weight])
