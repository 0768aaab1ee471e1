"""The device twin of the input generator draws the same bits as the host twin."""
import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu


def test_device_and_host_twins_agree():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    k = synth.key(0, 5)
    n = 3_000_001
    t = torch.empty(n, dtype=torch.int16, device="cuda")
    synth.dev_normal_bf16(k, 1234, n, 0.02, t.data_ptr(), torch.cuda.current_stream().cuda_stream)
    f = torch.empty(n, dtype=torch.float32, device="cuda")
    synth.dev_normal_f32(k, 99, n, 0.01, f.data_ptr(), torch.cuda.current_stream().cuda_stream)
    u = torch.empty(n, dtype=torch.int32, device="cuda")
    synth.dev_uniform_int(k, 7, n, 128000, u.data_ptr(), torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert np.array_equal(t.cpu().numpy().view(np.uint16), synth.normal_bf16(k, 1234, n, 0.02))
    assert np.array_equal(f.cpu().numpy().view(np.uint32), synth.normal_f32(k, 99, n, 0.01).view(np.uint32))
    assert np.array_equal(u.cpu().numpy(), synth.uniform_int(k, 7, n, 128000))
