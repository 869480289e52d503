"""The device twin of the weight generator draws the host recipe's exact bits."""
import numpy as np
import pytest
import torch

from synth import draws as D, device as SD

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("outliers", [None, (0.003, 10.0, 49.0)])
def test_device_draws_equal_host(outliers):
    shape = (5, 96, 512)
    host = D.expert_weights(0, 2, shape, start_row=123, rows=200, outliers=outliers)
    dev = torch.empty((200, 512), dtype=torch.float32, device="cuda")
    SD.expert_weights_into(dev, 0, 2, start_row=123, outliers=outliers)
    torch.cuda.synchronize()
    assert np.array_equal(dev.cpu().numpy().view(np.uint32), host.view(np.uint32))
