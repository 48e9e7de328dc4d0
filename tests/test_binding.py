"""Host-side checks of the Python binding that need no GPU: a call is refused when its tensors
are not on the current CUDA device (the library launches on the current device, and the
tensor maps of the tensor-core path would otherwise cover another GPU's memory)."""
import pytest
import torch

import gated_delta_rule_looped_b200 as lt2


class FakeTensor:
    """Just enough of a tensor for the binding's checks (shape and device); never read."""

    def __init__(self, shape, device, dtype=torch.bfloat16):
        self.shape = torch.Size(shape)
        self.device = torch.device(device)
        self.is_cuda = self.device.type == "cuda"
        self.dtype = dtype

    def dim(self):
        return len(self.shape)


def _call(dev):
    q = FakeTensor((1, 1, 1, 4, 8), dev)
    a = FakeTensor((1, 1, 1, 4), dev, torch.float32)
    return lt2._check_call(q, q, q, a, a, [], None, False, None)


def test_tensors_off_the_current_device_are_refused(monkeypatch):
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)
    with pytest.raises(ValueError, match="current device"):
        _call("cuda:1")


def test_host_tensors_are_refused(monkeypatch):
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)
    with pytest.raises(ValueError, match="CUDA tensor"):
        _call("cpu")
