"""Host-side argument checks of HostStreamer (no GPU work)."""
import pytest
import torch


def test_streamer_rejects_bad_sizes():
    from w8a8_linear_layers_b200.host import HostStreamer
    with pytest.raises(ValueError):
        HostStreamer("cpu", 0, 16, 16, torch.bfloat16, torch.bfloat16)
    with pytest.raises(ValueError):
        HostStreamer("cpu", 16, 16, 16, torch.bfloat16, torch.bfloat16, slots=1)
