"""The binding calls the library on the tensors' device and stream (no GPU).

The library launches on the current CUDA device and caches per-device
properties, so a call on tensors of another device must make that device
current for the duration of the call, and its default stream must be that
device's. These tests replace torch's CUDA namespace and the library by fakes
that record the current device each entry point sees.
"""
import contextlib
import types

import pytest
import torch

import w4a4_mxfp4_post_b200 as kq


class FakeStream:
    def __init__(self, index):
        self.device = torch.device("cuda", index)
        self.cuda_stream = 0x1000 + index


class FakeCuda:
    Stream = FakeStream

    def __init__(self):
        self.cur = 0
        self.switches = 0

    def current_device(self):
        return self.cur

    @contextlib.contextmanager
    def device(self, dev):
        prev, self.cur = self.cur, dev.index
        self.switches += 1
        try:
            yield
        finally:
            self.cur = prev

    def current_stream(self, device=None):
        return FakeStream(self.cur if device is None else device.index)


class FakeLib:
    def __init__(self, cuda, status=0):
        self.cuda, self.status, self.seen = cuda, status, []

    def __getattr__(self, name):
        if name == "kq_last_error":
            return lambda: b"fake failure"

        def entry(*args):
            self.seen.append((name, self.cuda.cur, args))
            return self.status

        return entry


@pytest.fixture
def fakes(monkeypatch):
    cuda = FakeCuda()
    fake_torch = types.SimpleNamespace(cuda=cuda)
    monkeypatch.setattr(kq, "_torch", lambda: fake_torch)
    fl = FakeLib(cuda)
    monkeypatch.setattr(kq, "lib", lambda: fl)
    return cuda, fl


def test_call_makes_the_tensors_device_current(fakes):
    cuda, fl = fakes
    kq._call("kq_quantize", torch.device("cuda", 1), 7)
    assert fl.seen == [("kq_quantize", 1, (7,))]
    assert cuda.cur == 0 and cuda.switches == 1


def test_call_on_the_current_device_does_not_switch(fakes):
    cuda, fl = fakes
    kq._call("mx_quantize", torch.device("cuda", 0))
    kq._call("kq_selftest_bounded_wait", None)
    assert [s[1] for s in fl.seen] == [0, 0]
    assert cuda.switches == 0


def test_call_error_restores_the_device_and_raises(fakes):
    cuda, fl = fakes
    fl.status = kq.KQ_ERR_SHAPE
    with pytest.raises(kq.KroQuantError) as e:
        kq._call("sq_quantize", torch.device("cuda", 2))
    assert e.value.status == kq.KQ_ERR_SHAPE and "fake failure" in str(e.value)
    assert fl.seen[0][1] == 2 and cuda.cur == 0


def test_default_stream_is_the_tensors_devices(fakes):
    assert kq._stream(None, torch.device("cuda", 3)).value == 0x1003
    assert kq._stream(None, None).value == 0x1000


def test_stream_of_another_device_is_refused(fakes):
    with pytest.raises(ValueError, match="stream is on"):
        kq._stream(FakeStream(0), torch.device("cuda", 1))
    assert kq._stream(FakeStream(1), torch.device("cuda", 1)).value == 0x1001


def test_raw_stream_handle_passes_through(fakes):
    assert kq._stream(0xBEEF, torch.device("cuda", 1)).value == 0xBEEF
