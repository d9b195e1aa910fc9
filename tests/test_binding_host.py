"""Argument checks of the Python binding that need no GPU: tensors of one call
on one device, caller workspaces on that device, streams of that device."""
import pytest
import torch

import global_gqa_b200 as g3


def test_on_device_rejects_a_tensor_elsewhere():
    cpu, meta = torch.device("cpu"), torch.device("meta")
    g3._on_device(cpu, a=torch.zeros(2), b=None)
    with pytest.raises(ValueError, match="must be on"):
        g3._on_device(cpu, a=torch.zeros(2), b=torch.zeros(2, device=meta))


def test_caller_workspace_must_be_on_the_call_device():
    with pytest.raises(ValueError, match="ws must be"):
        g3._ws(torch.zeros(1024, dtype=torch.uint8), 512, torch.device("meta"))
    with pytest.raises(ValueError, match="ws must be"):
        g3._ws(torch.zeros(64, 64, dtype=torch.uint8).t(), 512, torch.device("cpu"))


def test_caller_workspace_size_is_counted_in_bytes():
    ws = torch.zeros(100, dtype=torch.float32)
    buf, nbytes = g3._ws(ws, 400, torch.device("cpu"))
    assert buf is ws and nbytes == 400


def test_stream_of_another_device_is_rejected():
    class FakeStream:
        device = torch.device("cuda", 1)
        cuda_stream = 0
    with pytest.raises(ValueError, match="stream belongs to"):
        g3._stream_ptr(FakeStream(), torch.device("cuda", 0))


class _FakeStream:
    def __init__(self, handle):
        self.cuda_stream = handle


class _FakeTorch:
    """The few torch calls the workspace cache makes, without a GPU."""
    uint8 = torch.uint8
    device = torch.device

    class cuda:  # noqa: N801 (mirrors torch.cuda)
        current = _FakeStream(0)

        @staticmethod
        def current_device():
            return 0

        @staticmethod
        def current_stream(device=None):
            return _FakeTorch.cuda.current

        @staticmethod
        def stream(s):
            import contextlib
            return contextlib.nullcontext()

    @staticmethod
    def empty(n, dtype, device):
        return torch.empty(n, dtype=dtype)  # stands in for the device buffer


def test_workspace_cache_is_per_device_and_stream(monkeypatch):
    monkeypatch.setattr(g3, "_torch", lambda: _FakeTorch)
    monkeypatch.setattr(g3, "_workspaces", {})
    a = g3.workspace(512, torch.device("cuda", 0))
    assert g3.workspace(256, "cuda") is a                       # "cuda" names the current device
    assert g3.workspace(512, "cuda:0", stream=_FakeStream(0)) is a  # the current stream, named
    b = g3.workspace(512, "cuda:0", stream=_FakeStream(7))
    assert b is not a                                            # another stream, another buffer
    assert g3.workspace(512, "cuda:0", tag="backward") is not a  # another tag, another buffer
    c = g3.workspace(4096, "cuda:0")
    assert c is not a and c.numel() >= 4096                      # grown on demand
    assert g3.workspace(100, "cuda:0") is c


def test_release_workspaces_drops_one_stream_or_all(monkeypatch):
    monkeypatch.setattr(g3, "_torch", lambda: _FakeTorch)
    monkeypatch.setattr(g3, "_workspaces", {})
    a = g3.workspace(512, "cuda:0")
    b = g3.workspace(512, "cuda:0", stream=_FakeStream(7))
    g3.workspace(512, "cuda:0", tag="decode", stream=_FakeStream(7))
    assert g3.release_workspaces(stream=_FakeStream(7)) == 2     # both tags of that stream
    assert g3.workspace(512, "cuda:0") is a                       # the other stream's buffer stays
    assert g3.workspace(512, "cuda:0", stream=_FakeStream(7)) is not b
    assert g3.release_workspaces() == 2 and g3._workspaces == {}
