"""moba_fwd_host (host buffers, per-KV-group copies overlapped with the kernels over several
streams) returns exactly what moba_fwd returns on the same inputs."""
import numpy as np
import pytest
import torch

import synth
from _harness import params, run_gpu

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("w", [
    synth.Workload("h_gqa", [1500, 700, 3000], 8, 2, 128, 256, 3, seed=41, rope_theta=500000.0, plant=0.5),
    synth.Workload("h_mha", [2049], 3, 3, 64, 128, 4, seed=42),
], ids=lambda w: w.name)
@pytest.mark.parametrize("nstreams", [1, 3])
def test_host_forward_equals_device_forward(w, nstreams, cuda_device):
    import block_sparse_attention_gate_b200 as mb
    Q, K, V = w.fill("q"), w.fill("k"), w.fill("v")
    ref = run_gpu(w, Q, K, V)
    p = params(w)
    pin = lambda a: torch.from_numpy(a.view(np.int16)).pin_memory().view(torch.bfloat16)
    Qh, Kh, Vh = pin(Q), pin(K), pin(V)
    Oh = torch.empty(Qh.shape, dtype=torch.bfloat16).pin_memory()
    Lh = torch.full((w.total_tokens, w.num_q_heads), -1.0, dtype=torch.float32).pin_memory()
    streams = [torch.cuda.Stream() for _ in range(nstreams)]
    staging = torch.empty(mb.moba_host_staging_size(p, nstreams), dtype=torch.uint8, device="cuda")
    mb.moba_fwd_host(p, Qh, Kh, Vh, Oh, Lh, staging, streams)
    for s in streams:
        s.synchronize()
    assert mb.moba_read_device_error(clear=True) == 0
    np.testing.assert_array_equal(Oh.float().numpy(), ref["O"])
    np.testing.assert_array_equal(Lh.numpy(), ref["LSE"])
