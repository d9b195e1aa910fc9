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
