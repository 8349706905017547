"""bench.py's timing helpers on the CPU, with a fake device clock: flushes stay outside the
timed intervals, and a stage is timed back to back only when one call reads more than L2
holds."""
import contextlib

import pytest

import bench


class _Clock:
    def __init__(self):
        self.t = 0.0
        self.log = []


@pytest.fixture
def clock(monkeypatch):
    c = _Clock()

    class FakeEvent:
        def __init__(self, enable_timing=False):
            assert enable_timing
            self.t = None

        def record(self, stream=None):
            self.t = c.t
            c.log.append("rec")

        def synchronize(self):
            pass

        def elapsed_time(self, other):
            return other.t - self.t

    monkeypatch.setattr(bench.torch.cuda, "Event", FakeEvent)
    monkeypatch.setattr(bench.torch.cuda, "stream", lambda s: contextlib.nullcontext())
    return c


def _call(c, ms=2.0):
    def f():
        c.t += ms
        c.log.append("call")
    return f


class _Flush:
    def __init__(self, c, ms=50.0):
        self.c, self.ms = c, ms

    def zero_(self):
        self.c.t += self.ms
        self.c.log.append("flush")


def test_back_to_back(clock):
    assert bench.timed_back_to_back(_call(clock), 4, None) == pytest.approx(8.0)
    assert clock.log == ["rec"] + ["call"] * 4 + ["rec"]


def test_flushed_excludes_the_flushes(clock):
    assert bench.timed_flushed(_call(clock), 3, None, _Flush(clock)) == pytest.approx(6.0)
    assert clock.log == ["flush", "rec", "call", "rec"] * 3


def test_stage_timing_picks_by_bytes(clock):
    big = bench.L2_BYTES + 1
    ms, how = bench.time_stage(_call(clock), 10, big, None, _Flush(clock))
    assert ms == pytest.approx(2.0) and "back to back" in how
    assert "flush" not in clock.log and clock.log.count("call") == 15       # 5 warm-up + 10 timed
    clock.log.clear()
    ms, how = bench.time_stage(_call(clock), 10, bench.L2_BYTES // 2, None, _Flush(clock))
    assert ms == pytest.approx(2.0) and "flushed" in how
    assert clock.log[:5] == ["call"] * 5 and clock.log[5:] == ["flush", "rec", "call", "rec"] * 10


def test_packed_buffer_views_are_aligned_disjoint_and_typed():
    import torch
    like = {"a": torch.zeros(3, 5, dtype=torch.bfloat16), "b": torch.zeros(7, dtype=torch.int32),
            "c": torch.zeros(2, 64, dtype=torch.uint8), "d": torch.zeros(1, dtype=torch.float32)}
    p = bench.Packed(like)
    spans = []
    for k, v in like.items():
        w = p.views[k]
        assert w.dtype == v.dtype and w.shape == v.shape and w.is_contiguous()
        off = w.data_ptr() - p.buf.data_ptr()
        assert off % 256 == 0
        spans.append((off, off + v.numel() * v.element_size()))
    spans.sort()
    assert all(a[1] <= b[0] for a, b in zip(spans, spans[1:]))
    assert p.nbytes == p.buf.numel() and spans[-1][1] <= p.nbytes
    for i, (k, v) in enumerate(like.items()):
        p.views[k].fill_(i + 1)
    for i, k in enumerate(like):
        assert torch.all(p.views[k] == i + 1)
