"""CPU checks of the Python binding's launch context: every call runs on its tensors'
device and on a stream of that device (the library plans and launches on the current
CUDA device, so a stream of another device would be a mismatch). No GPU is needed:
the streams are stand-ins."""
import pytest
import torch

import selective_state_space_47_b200 as ssm


class _FakeStream:
    def __init__(self, device, handle):
        self.device = torch.device(device)
        self.cuda_stream = handle


def test_stream_of_another_device_is_refused():
    with pytest.raises(ValueError):
        ssm._resolve_stream(_FakeStream("cuda:1", 7), torch.device("cuda:0"))


def test_caller_stream_of_the_same_device_is_used():
    s = _FakeStream("cuda:1", 7)
    assert ssm._resolve_stream(s, torch.device("cuda:1")) is s
    assert ssm._handle(s).value == 7


def test_default_stream_is_the_tensors_devices(monkeypatch):
    asked = []

    def fake_current_stream(device=None):
        asked.append(device)
        return _FakeStream(device, 42)

    monkeypatch.setattr(torch.cuda, "current_stream", fake_current_stream)
    s = ssm._resolve_stream(None, torch.device("cuda:3"))
    assert asked == [torch.device("cuda:3")]
    assert s.device == torch.device("cuda:3") and s.cuda_stream == 42
