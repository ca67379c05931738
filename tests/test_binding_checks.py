"""Host-side argument checks of the binding that need no GPU.

The library launches on the calling thread's current CUDA device and takes
raw pointers, so the binding refuses tensors and streams of another device and
status words that are not one int32 word in device memory.  CUDA's device
query is replaced by a fake here; nothing is launched.
"""
from types import SimpleNamespace

import pytest
import torch

from future_attention_targets_b200 import _binding as B


@pytest.fixture
def current_device_0(monkeypatch):
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)


def test_tensor_on_another_device_is_refused(current_device_0):
    B._on_current_device(SimpleNamespace(device=torch.device("cuda", 0)), "q")
    with pytest.raises(ValueError, match="current CUDA device is cuda:0"):
        B._on_current_device(SimpleNamespace(device=torch.device("cuda", 1)), "q")


def test_stream_of_another_device_is_refused(current_device_0):
    ok = SimpleNamespace(device=torch.device("cuda", 0), cuda_stream=0x1234)
    assert B._stream_ptr(ok) == 0x1234
    with pytest.raises(ValueError, match="stream belongs to cuda:1"):
        B._stream_ptr(SimpleNamespace(device=torch.device("cuda", 1), cuda_stream=0x1234))
    assert B._stream_ptr(0x5678) == 0x5678                  # a raw handle is passed through


def test_status_word_checks():
    dev = torch.device("cuda", 0)
    assert B._status_ptr(None, dev) is None
    for bad in (torch.zeros(1, dtype=torch.int32),          # host memory
                torch.zeros(1, dtype=torch.float32),
                torch.zeros(0, dtype=torch.int32),
                "not a tensor"):
        with pytest.raises(ValueError, match="status"):
            B._status_ptr(bad, dev)
