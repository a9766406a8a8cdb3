"""Host-buffer prefill (x and y in host memory, copies overlapped with the row-separable
stages) against the device-buffer prefill and the oracle."""
import numpy as np
import pytest
import torch

from differential_latent_attention_fwd_b200 import binding as gb
from tests.gpu_helpers import check, oracle_prefill, prefill_case, to_np

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,T,window,pieces,pinned", [
    (1, 2048, 0, 8, True),
    (2, 700, 128, 3, True),
    (1, 513, 0, 1, True),
    (1, 1000, 0, 64, False),      # pageable memory: same result, copies not overlapped
])
def test_host_prefill_matches_device_prefill(cuda_ok, B, T, window, pieces, pinned):
    shape, inp, layer, x = prefill_case(B, T, window, seed=29)
    y_dev = layer.prefill(x)
    torch.cuda.synchronize()
    x_host = inp.x.contiguous()
    if pinned:
        x_host = x_host.pin_memory()
    y_host = torch.empty_like(x_host)
    if pinned:
        y_host = y_host.pin_memory()
    layer.prefill_host(x_host, y_host, n_pieces=pieces)
    torch.cuda.synchronize()
    assert gb.gdla_device_error() == 0
    errs = []
    check("host-buffer vs device-buffer prefill", to_np(y_host), to_np(y_dev), rel=1e-3, mabs=5e-3, errors=errs)
    rows = sorted(set([0, T - 1] + list(np.linspace(0, T - 1, 12).astype(int))))
    yo = oracle_prefill(inp, rows=rows)
    for b in range(B):
        check(f"host-buffer prefill vs oracle b={b}", to_np(y_host[b, rows]), yo[b], errors=errs)
    assert not errs, "\n".join(errs)


def test_host_prefill_rejects_device_tensors(cuda_ok):
    shape, inp, layer, x = prefill_case(1, 64, 0, seed=2)
    with pytest.raises(ValueError):
        layer.prefill_host(x)
