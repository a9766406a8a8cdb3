"""The C ABI library loads and exports every entry point declared in include/gdla.h, and its
host-side validation answers without a GPU (no kernel is launched here)."""
import ctypes

import pytest

from differential_latent_attention_fwd_b200 import binding as gb
from differential_latent_attention_fwd_b200 import build as gbuild
from differential_latent_attention_fwd_b200.synth import GdlaShape


@pytest.fixture(scope="module")
def L():
    gbuild.build()
    return gb.lib()


def test_every_declared_symbol_is_exported(L):
    names = gb.header_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(L, n), f"{n} declared in gdla.h but not exported"


def test_status_strings(L):
    for code in range(0, -7, -1):
        assert gb.gdla_status_string(code) not in ("", "unknown status")
    assert gb.gdla_status_string(-99) == "unknown status"


def test_workspace_size_and_offsets(L):
    cfg = gb.make_config(GdlaShape())
    n = gb.gdla_workspace_size(cfg, 1, 256, gb.GDLA_MODE_PREFILL)
    M = 256
    # dominant buffers: q^C|q^R (fp16), gate, Dg, K|V, noise outputs, fp32 down-projection
    assert n >= M * (80 * 192 * 2 + 8192 * 2 * 2 + 4096 * 2 + 16 * 128 * 4 + 1664 * 4)
    offs = [gb.gdla_workspace_offset(cfg, 1, 256, 0, i) for i in range(10)]
    assert offs == sorted(offs) and all(o % 256 == 0 for o in offs) and offs[-1] < n
    assert gb.gdla_workspace_size(cfg, 2, 256, 0) > n
    d = gb.gdla_workspace_size(cfg, 64, 1, gb.GDLA_MODE_DECODE)
    assert d > 64 * 80 * 576 * 2
    # W_UK^T, then [W_a^Q | W_a^KV | W^lambda] and [W_b^Q | W^G], each rounded up to 256 bytes
    r256 = lambda b: (b + 255) // 256 * 256
    assert gb.gdla_absorbed_size(cfg) == (r256(16 * 128 * 512 * 2) + r256(4096 * 1664 * 2) +
                                          r256(1024 * (80 * 192 + 64 * 128) * 2))


def test_host_validation_without_gpu(L):
    cfg = gb.make_config(GdlaShape())
    bad = gb.make_config(GdlaShape(d_nope=64))
    with pytest.raises(gb.GdlaError) as e:
        gb.gdla_workspace_size(bad, 1, 16, 0)
    assert e.value.status == -2
    with pytest.raises(gb.GdlaError) as e:
        gb.gdla_workspace_size(cfg, 0, 16, 0)
    assert e.value.status == -1
    with pytest.raises(gb.GdlaError) as e:
        gb.gdla_workspace_size(cfg, 1, 16, 7)
    assert e.value.status == -1
    # null weights / buffers are rejected before any launch
    w = gb.gdla_weights_t()
    rc = L.gdla_prefill_fwd(ctypes.byref(cfg), ctypes.byref(w), None, 1, 16, None, None, 0, None, 0, None)
    assert rc == -1
    rc = L.gdla_decode_fwd(ctypes.byref(cfg), None, None, None, None, 1, 1, None, None, 0, None)
    assert rc == -1
    # an absorbed handle that was never filled is rejected
    ab = gb.gdla_absorbed_t()
    rc = L.gdla_decode_fwd(ctypes.byref(cfg), ctypes.byref(ab), None, None, None, 1, 1, None, None, 0, None)
    assert rc == -1
    # GDA-style config (g = 1) is outside the compiled specialisation
    gda = gb.make_config(GdlaShape(n_signal=16, n_noise=16))
    with pytest.raises(gb.GdlaError) as e:
        gb.gdla_workspace_size(gda, 1, 16, 0)
    assert e.value.status == -2


def test_misaligned_pointer_rejected(L):
    cfg = gb.make_config(GdlaShape())
    fake = ctypes.c_void_p(0x1000)
    w = gb.gdla_weights_t(fake, fake, fake, fake, fake, fake, fake, None, None)
    rc = L.gdla_prefill_fwd(ctypes.byref(cfg), ctypes.byref(w), ctypes.c_void_p(0x1008), 1, 16,
                            fake, None, 0, fake, 1 << 40, None)
    assert rc == -1
    # workspace too small is reported before anything touches the device
    rc = L.gdla_prefill_fwd(ctypes.byref(cfg), ctypes.byref(w), fake, 1, 16, fake, None, 0, fake, 16, None)
    assert rc == -3


def test_context_entry_points_validate_on_the_host(L):
    cfg = gb.make_config(GdlaShape())
    fake = ctypes.c_void_p(0x1000)
    w = gb.gdla_weights_t(fake, fake, fake, fake, fake, fake, fake, None, None)
    # context workspace covers prefix + local rows, like a prefill of that many tokens
    assert gb.gdla_workspace_size(cfg, 1, 300, gb.GDLA_MODE_CONTEXT) == gb.gdla_workspace_size(cfg, 1, 300, 0)
    big = 1 << 40
    # a prefix longer than the position offset
    rc = L.gdla_prefill_context_fwd(ctypes.byref(cfg), ctypes.byref(w), fake, 16, 8, fake, 16, fake, None,
                                    fake, big, None)
    assert rc == -1
    # prefix rows announced but no pointer
    rc = L.gdla_prefill_context_fwd(ctypes.byref(cfg), ctypes.byref(w), fake, 16, 16, None, 16, fake, None,
                                    fake, big, None)
    assert rc == -1
    # workspace sized for the local tokens only
    small = gb.gdla_workspace_size(cfg, 1, 16, 0)
    rc = L.gdla_prefill_context_fwd(ctypes.byref(cfg), ctypes.byref(w), fake, 16, 512, fake, 512, fake, None,
                                    fake, small, None)
    assert rc == -3
    # latent-only call: negative offset, null output
    rc = L.gdla_latent_fwd(ctypes.byref(cfg), ctypes.byref(w), fake, 16, -1, fake, fake, big, None)
    assert rc == -1
    rc = L.gdla_latent_fwd(ctypes.byref(cfg), ctypes.byref(w), fake, 16, 0, None, fake, big, None)
    assert rc == -1


def test_training_entry_points_validate_on_the_host(L):
    cfg = gb.make_config(GdlaShape())
    fake = ctypes.c_void_p(0x1000)
    odd = ctypes.c_void_p(0x1002)
    f, b = ctypes.c_size_t(0), ctypes.c_size_t(0)
    assert L.gdla_attn_train_workspace_size(ctypes.byref(cfg), 0, 16, ctypes.byref(f), ctypes.byref(b)) == -1
    assert L.gdla_attn_train_workspace_size(ctypes.byref(cfg), 1, 16, None, ctypes.byref(b)) == -1
    sizes = []
    for T in (16, 600, 1200):
        assert L.gdla_attn_train_workspace_size(ctypes.byref(cfg), 1, T, ctypes.byref(f), ctypes.byref(b)) == 0
        assert f.value > 0 and b.value > 0
        sizes.append(b.value)
    assert sizes[0] < sizes[1] < sizes[2]   # the backward's score buffers grow with T
    big = 1 << 40
    fwd = lambda *a: L.gdla_attn_train_fwd(ctypes.byref(cfg), *a)
    # qq, kv, kr16, lam, gate, B, T, dg_out, h_out, lse_out, ws, ws_bytes, stream
    assert fwd(None, fake, fake, fake, fake, 1, 16, fake, fake, fake, fake, big, None) == -1
    assert fwd(fake, fake, odd, fake, fake, 1, 16, fake, fake, fake, fake, big, None) == -1
    assert fwd(fake, fake, fake, fake, fake, 1, 0, fake, fake, fake, fake, big, None) == -1
    assert fwd(fake, fake, fake, fake, fake, 1, 16, fake, fake, fake, fake, 16, None) == -3
    bwd = lambda *a: L.gdla_attn_bwd(ctypes.byref(cfg), *a)
    # qq, kv, kr16, lam, gate, h, lse, d_dg, B, T, d_qq, d_kv, d_kr, d_lam, d_gate, ws, ws_bytes, stream
    ok8 = [fake] * 8
    outs = [fake] * 5
    assert bwd(*([None] + ok8[1:]), 1, 16, *outs, fake, big, None) == -1
    assert bwd(*ok8, 1, 16, *(outs[:4] + [odd]), fake, big, None) == -1
    assert bwd(*ok8, -1, 16, *outs, fake, big, None) == -1
    assert bwd(*ok8, 1, 16, *outs, fake, 16, None) == -3


def test_binding_rejects_wrong_tensors_before_the_library():
    """Argument marshalling refuses host tensors where device memory is expected (and the
    reverse), wrong dtypes and non-contiguous views; nothing reaches the C ABI."""
    import pytest
    import torch
    cfg = gb.make_config(GdlaShape())
    dev_like = torch.zeros(16, dtype=torch.float16)          # a host tensor: refused as device memory
    with pytest.raises(ValueError):
        gb.gdla_attn_train_fwd(cfg, dev_like, dev_like, dev_like, torch.zeros(4), torch.zeros(4).bfloat16(),
                               1, 16, None, None, None, torch.zeros(16, dtype=torch.uint8))
    with pytest.raises(TypeError):
        gb.gdla_attn_train_fwd(cfg, torch.zeros(16), dev_like, dev_like, torch.zeros(4),
                               torch.zeros(4).bfloat16(), 1, 16, None, None, None, torch.zeros(16, dtype=torch.uint8))
    with pytest.raises(TypeError):
        gb._ptr([1, 2, 3], None, "x")
    with pytest.raises(ValueError):
        gb._host_ptr(torch.zeros(8, 8).t(), torch.float32, "x")   # non-contiguous
    with pytest.raises(TypeError):
        gb._host_ptr(torch.zeros(8), torch.bfloat16, "x")
    assert gb._host_ptr(torch.zeros(8, dtype=torch.bfloat16), torch.bfloat16, "x").value is not None


def test_fp8_row_bytes_matches_header():
    from oracle import gdla_oracle as O
    assert gb.FP8_ROW_BYTES == gb._header_define("GDLA_FP8_ROW_BYTES") == O.fp8_row_bytes(576)
