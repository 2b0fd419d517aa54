"""The binding's two-green-context split (GreenPartition) on the host, against
a fake of the driver calls it makes: the SM resource is split once, the
dispatch group and the remainder each get a green context and one stream,
close() releases both, and a driver error part way releases whatever was
already created. No GPU: the fake stands in for cuda.bindings.driver."""
import types

import pytest

from combine_softmax_top_b200 import moe


class _FakeDriver:
    def __init__(self, sms=148, granularity=8, fail_ctx_at=None):
        self.sms, self.gran, self.fail_ctx_at = sms, granularity, fail_ctx_at
        self.log = []
        self.live_ctx, self.live_streams = set(), set()
        ok = object()
        self.CUresult = types.SimpleNamespace(CUDA_SUCCESS=ok, CUDA_ERROR_INVALID_VALUE=object())
        self._ok = ok
        self.CUdevResourceType = types.SimpleNamespace(CU_DEV_RESOURCE_TYPE_SM=1)
        self.CUgreenCtxCreate_flags = types.SimpleNamespace(CU_GREEN_CTX_DEFAULT_STREAM=1)
        self.CUstream_flags = types.SimpleNamespace(CU_STREAM_NON_BLOCKING=1)
        self._next = 1000

    @staticmethod
    def _res(n):
        return types.SimpleNamespace(sm=types.SimpleNamespace(smCount=n))

    def cuInit(self, flags):
        return (self._ok,)

    def cuDeviceGet(self, index):
        self.log.append(("device", index))
        return (self._ok, index)

    def cuDeviceGetDevResource(self, dev, kind):
        return (self._ok, self._res(self.sms))

    def cuDevSmResourceSplitByCount(self, n_groups, res, flags, min_count):
        n = -(-min_count // self.gran) * self.gran
        self.log.append(("split", n_groups, min_count, n))
        return (self._ok, [self._res(n)], 1, self._res(res.sm.smCount - n))

    def cuDevResourceGenerateDesc(self, resources, n):
        return (self._ok, ("desc", resources[0].sm.smCount))

    def cuGreenCtxCreate(self, desc, dev, flags):
        made = len([e for e in self.log if e[0] == "ctx"])
        if self.fail_ctx_at is not None and made == self.fail_ctx_at:
            return (self.CUresult.CUDA_ERROR_INVALID_VALUE, None)
        self._next += 1
        self.log.append(("ctx", desc[1], self._next))
        self.live_ctx.add(self._next)
        return (self._ok, self._next)

    def cuGreenCtxStreamCreate(self, ctx, flags, prio):
        self._next += 1
        self.log.append(("stream", ctx, prio, self._next))
        self.live_streams.add(self._next)
        return (self._ok, self._next)

    def cuStreamSynchronize(self, st):
        self.log.append(("sync", st))
        return (self._ok,)

    def cuStreamDestroy(self, st):
        self.live_streams.discard(st)
        return (self._ok,)

    def cuGreenCtxDestroy(self, ctx):
        self.live_ctx.discard(ctx)
        return (self._ok,)


@pytest.fixture
def fake_driver(monkeypatch):
    import cuda.bindings
    def install(**kw):
        drv = _FakeDriver(**kw)
        monkeypatch.setattr(cuda.bindings, "driver", drv, raising=False)
        return drv
    return install


def test_two_disjoint_partitions_and_release(fake_driver):
    drv = fake_driver()
    gp = moe.GreenPartition(20, 3)
    assert ("device", 3) in drv.log
    assert [e for e in drv.log if e[0] == "split"] == [("split", 1, 20, 24)]   # one split, rounded up
    assert (gp.dispatch_sms, gp.main_sms) == (24, 124)
    assert gp.dispatch_sms + gp.main_sms == drv.sms                           # disjoint, covering
    ctx = [e for e in drv.log if e[0] == "ctx"]
    assert [c[1] for c in ctx] == [24, 124]
    streams = [e for e in drv.log if e[0] == "stream"]
    # dispatch's stream in the dispatch context at high priority, the layer's in the other
    assert (streams[0][1], streams[0][2]) == (ctx[0][2], -1)
    assert (streams[1][1], streams[1][2]) == (ctx[1][2], 0)
    assert (gp.dispatch_stream, gp.main_stream) == (streams[0][3], streams[1][3])
    gp.close()
    assert not drv.live_ctx and not drv.live_streams
    assert {e[1] for e in drv.log if e[0] == "sync"} == {streams[0][3], streams[1][3]}
    gp.close()                                                               # idempotent


def test_failure_releases_what_was_made(fake_driver):
    drv = fake_driver(fail_ctx_at=1)                 # the second green context fails
    with pytest.raises(RuntimeError, match="cuGreenCtxCreate"):
        moe.GreenPartition(8, 0)
    assert len([e for e in drv.log if e[0] == "ctx"]) == 1
    assert not drv.live_ctx and not drv.live_streams
