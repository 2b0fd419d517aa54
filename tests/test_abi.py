"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point include/moe.h declares, sizes workspaces and rejects bad
arguments before touching CUDA."""
import ctypes
import os
import re

import pytest

from combine_softmax_top_b200 import moe
from combine_softmax_top_b200 import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    return sorted(set(re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", src)))


def test_header_declares_the_python_exports():
    assert _declared() == sorted(moe.EXPORTS)


def test_library_exports_every_declared_symbol():
    L = moe.lib()
    for name in _declared():
        assert hasattr(L, name), name


def test_status_strings():
    for code in range(7):
        assert moe.moe_status_string(code)
    assert moe.moe_status_string(99) == "unknown status"


@pytest.mark.parametrize("name", ["tiny", "decode", "prefill", "skew", "sweep"])
def test_workspace_bytes(name):
    s = W.spec(name)
    n = moe.moe_workspace_bytes(moe.make_shape(s))
    assert n > 256 and n % 256 == 0


def test_workspace_grows_with_capacity():
    s = W.spec("decode")
    a = moe.moe_workspace_bytes(moe.make_shape(s))
    b = moe.moe_workspace_bytes(moe.make_shape(s.with_(cap_rows=1024)))
    assert b > a


@pytest.mark.parametrize("field,value", [
    ("topk", 0), ("topk", 33), ("E", 0), ("H", 100), ("quant_block", 64), ("flags", 4),
    ("cap_rows", 100), ("renorm", 2), ("T", -1), ("act_dtype", 7),
])
def test_invalid_shapes_rejected_on_host(field, value):
    sh = moe.make_shape(W.spec("decode"))
    setattr(sh, field, value)
    n = ctypes.c_size_t(0)
    assert moe.lib().moe_workspace_bytes(ctypes.byref(sh), ctypes.byref(n)) == 1
    # every entry point checks the shape first, before any CUDA call
    assert moe.lib().moe_route(ctypes.byref(sh), None, None, None, None, None) == 1


@pytest.mark.parametrize("base,over", [
    ("sweep", {}),                          # identity experts have no FFN to share
    ("decode", {"topk": 32}),               # topk + 1 slots > 32
    ("decode", {"cap_rows": 0, "T": 200}),  # placeholder: cap set below T
])
def test_shared_expert_preconditions(base, over):
    """The shared expert takes every token (cap >= T), one more slot per token
    (topk + 1 <= 32), and needs real experts."""
    sh = moe.make_shape(W.spec(base, shared=1))
    for f, v in over.items():
        setattr(sh, f, v)
    if "T" in over:
        sh.cap_rows = 128                   # 128 < T = 200
    n = ctypes.c_size_t(0)
    assert moe.lib().moe_workspace_bytes(ctypes.byref(sh), ctypes.byref(n)) == 1


def test_shared_expert_workspace_covers_one_more_expert():
    s = W.spec("decode")
    a = moe.moe_workspace_bytes(moe.make_shape(s))
    b = moe.moe_workspace_bytes(moe.make_shape(s.with_(shared=1)))
    assert b > a


@pytest.mark.parametrize("over", [
    {"cap_rows": 128},   # the counting pass sizes the windows
    {"T": 1 << 20},      # more than 65535 tiles of 128 rows
])
def test_compact_windows_preconditions(over):
    sh = moe.make_shape(W.spec("prefill", compact=1))
    for f, v in over.items():
        setattr(sh, f, v)
    n = ctypes.c_size_t(0)
    assert moe.lib().moe_workspace_bytes(ctypes.byref(sh), ctypes.byref(n)) == 1


def test_compact_windows_rows_and_workspace():
    """Compact windows: the buffers hold T * k rows plus one partial tile per
    expert instead of E windows of round_up(T, 128) rows; the workspace's
    per-tile arrays shrink with them."""
    s = W.spec("prefill")
    c = s.with_(compact=1)
    assert c.rows() == (8192 * 8 // 128 + 256) * 128 < s.rows() // 20
    assert moe.moe_workspace_bytes(moe.make_shape(c)) < moe.moe_workspace_bytes(moe.make_shape(s))
    sc = c.with_(shared=1)
    assert sc.rows() == (-(-8192 * 9 // 128) + 257) * 128
    assert moe.moe_workspace_bytes(moe.make_shape(sc)) > 0


def test_unsupported_dtype_combination():
    sh = moe.make_shape(W.spec("decode"))
    sh.h_dtype = moe.MOE_BF16   # fp8 weights with a bf16 h is not a supported layer
    n = ctypes.c_size_t(0)
    assert moe.lib().moe_workspace_bytes(ctypes.byref(sh), ctypes.byref(n)) == 2


def test_null_shape_and_output():
    n = ctypes.c_size_t(0)
    assert moe.lib().moe_workspace_bytes(None, ctypes.byref(n)) == 1
    sh = moe.make_shape(W.spec("tiny"))
    assert moe.lib().moe_workspace_bytes(ctypes.byref(sh), None) == 1
    assert moe.lib().moe_poll_status(None, None) == 1


def test_noalloc_dispatch_refuses_compact_windows():
    """The no-workspace dispatch has no room for the counting pass: the
    compact flag is refused before any pointer is looked at."""
    sh = moe.make_shape(W.spec("decode", compact=1))
    assert moe.lib().moe_dispatch_noalloc(ctypes.byref(sh), None, None, None, None) == 2


def test_fp4_weight_layer_shape_accepted_and_e2m1_only_for_weights():
    """MX FP4 (E2M1) is a weight dtype: the fp4-weight layer (bf16 x, e4m3
    tokens and h, E2M1 weights) is accepted; E2M1 anywhere else is refused."""
    sh = moe.make_shape(W.spec("decode_fp4"))
    n = ctypes.c_size_t(0)
    assert moe.lib().moe_workspace_bytes(ctypes.byref(sh), ctypes.byref(n)) == 0 and n.value > 0
    for field in ("act_dtype", "xq_dtype", "h_dtype", "y_dtype", "out_dtype"):
        bad = moe.make_shape(W.spec("decode_fp4"))
        setattr(bad, field, moe.MOE_E2M1)
        assert moe.lib().moe_workspace_bytes(ctypes.byref(bad), ctypes.byref(n)) in (1, 2), field


@pytest.mark.parametrize("n,rows,cols", [(1, 100, 128), (1, 128, 96), (-1, 128, 128)])
def test_pack_mx_scales_rejects_bad_sizes(n, rows, cols):
    """Sizes are checked on the host, before any pointer is used."""
    assert moe.lib().moe_pack_mx_scales(n, rows, cols, None, None, None) == 1


def test_pack_mx_scales_empty_enqueues_nothing():
    assert moe.lib().moe_pack_mx_scales(0, 128, 128, None, None, None) == 0


def test_layer_workspace_holds_the_intermediates():
    """moe_layer keeps topk_idx/topk_w, the expert-major buffers and y after
    the stage workspace: its size is at least the stage workspace plus those
    arrays at the sizes moe.h gives for them."""
    for s in (W.spec("decode"), W.spec("prefill", compact=1), W.spec("tiny"), W.spec("sweep"),
              W.spec("decode", shared=1)):
        sh = moe.make_shape(s)
        stage = moe.moe_workspace_bytes(sh)
        layer = moe.moe_layer_workspace_bytes(sh)
        el = {"f32": 4, "bf16": 2, "e4m3": 1}
        rows = s.rows()
        need = 2 * s.T * s.ks * 4 + rows * s.H * el[s.xq] + rows * 4 + s.T * s.ks * 4
        if not s.identity:
            need += rows * s.I * el[s.h] + rows * s.H * el[s.y]
        assert layer >= stage + need, s.name
        assert layer % 256 == 0


def test_layer_checks_arguments_before_any_launch():
    sh = moe.make_shape(W.spec("decode"))
    L = moe.lib()
    assert L.moe_layer(ctypes.byref(sh), None, None, None, None, None, None) == 1
    bad = moe.make_shape(W.spec("decode"))
    bad.topk = 0
    n = ctypes.c_size_t(0)
    assert L.moe_layer_workspace_bytes(ctypes.byref(bad), ctypes.byref(n)) == 1
    assert L.moe_layer_workspace_bytes(ctypes.byref(sh), None) == 1


def test_overlap_checks_its_partition_before_any_cuda_call():
    """moe_layer_overlap refuses a missing overlap description, a missing
    stream or event, the dispatch stream equal to the layer's stream, and an
    empty dispatch partition, all on the host."""
    sh = moe.make_shape(W.spec("decode"))
    L = moe.lib()
    fake = ctypes.c_void_p(1 << 20)
    w = moe.moe_weights()
    assert L.moe_layer_overlap(ctypes.byref(sh), fake, fake, ctypes.byref(w), fake, fake, None, None) == 1

    def ov(**kw):
        o = moe.moe_overlap()
        o.dispatch_stream, o.fork_event, o.join_event, o.dispatch_sms, o.ffn_sms = 1 << 12, 1 << 13, 1 << 14, 20, 0
        for k, v in kw.items():
            setattr(o, k, v)
        return o

    for bad in (dict(dispatch_stream=0), dict(fork_event=0), dict(join_event=0), dict(dispatch_sms=0),
                dict(dispatch_sms=-3), dict(ffn_sms=-1), dict(dispatch_stream=1 << 16)):
        o = ov(**bad)
        stream = ctypes.c_void_p(1 << 16)       # the last case: the same stream twice
        assert L.moe_layer_overlap(ctypes.byref(sh), fake, fake, ctypes.byref(w), fake, fake, stream,
                                   ctypes.byref(o)) == 1, bad
    bad = moe.make_shape(W.spec("decode"))
    bad.topk = 0
    o = ov()
    assert L.moe_layer_overlap(ctypes.byref(bad), fake, fake, ctypes.byref(w), fake, fake, None,
                               ctypes.byref(o)) == 1
