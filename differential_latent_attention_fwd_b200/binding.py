"""ctypes binding of libgdla.so (include/gdla.h): argument marshalling only.

Every function here has the name of the C entry point it wraps, takes torch tensors (device
memory owned by the caller) or plain integers, checks dtype/device/contiguity, and forwards raw
pointers.  All arithmetic happens in the CUDA kernels behind the C ABI; if the library is
missing this module raises instead of falling back to anything else.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libgdla.so")
HEADER = os.path.join(HERE, "..", "include", "gdla.h")

GDLA_MODE_PREFILL = 0
GDLA_MODE_DECODE = 1
GDLA_MODE_VARLEN = 2
GDLA_MODE_CONTEXT = 3
GDLA_MODE_HOST = 4
STATUS = {0: "GDLA_OK", -1: "GDLA_ERR_INVALID_ARG", -2: "GDLA_ERR_UNSUPPORTED_SHAPE",
          -3: "GDLA_ERR_WORKSPACE_TOO_SMALL", -4: "GDLA_ERR_LAUNCH",
          -5: "GDLA_ERR_DEVICE_TIMEOUT", -6: "GDLA_ERR_CUDA",
          -7: "GDLA_ERR_DEVICE_DATA"}


class GdlaError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} -> {status} ({STATUS.get(status, '?')})")
        self.status = status


class gdla_config_t(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("d_model", "q_rank", "kv_rank", "n_signal", "n_noise",
                                             "n_kv_heads", "d_nope", "d_rope", "d_v", "window")] + \
               [("rope_theta", ctypes.c_float), ("rms_eps", ctypes.c_float)]


class gdla_weights_t(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("W_aQ", "W_bQ", "W_aKV", "W_bKV", "W_lambda", "W_G",
                                                "W_O", "g_q", "g_kv")]


class gdla_absorbed_t(ctypes.Structure):
    _fields_ = [("w", gdla_weights_t), ("W_UKt", ctypes.c_void_p), ("W_a", ctypes.c_void_p),
                ("W_bqg", ctypes.c_void_p), ("cfg", gdla_config_t),
                ("magic", ctypes.c_uint32)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libgdla.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing; build it with "
                               "`python -m differential_latent_attention_fwd_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I, SZ, ULL = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_ulonglong
        cfgp, wp, abp = (ctypes.POINTER(gdla_config_t), ctypes.POINTER(gdla_weights_t),
                         ctypes.POINTER(gdla_absorbed_t))
        sig = {
            "gdla_workspace_size": [cfgp, I, I, I, ctypes.POINTER(SZ)],
            "gdla_absorbed_size": [cfgp, ctypes.POINTER(SZ)],
            "gdla_prefill_fwd": [cfgp, wp, P, I, I, P, P, I, P, SZ, P],
            "gdla_absorb_weights": [cfgp, wp, P, SZ, abp, P],
            "gdla_decode_fwd": [cfgp, abp, P, P, P, I, I, P, P, SZ, P],
            "gdla_device_error": [P, ctypes.POINTER(I), I],
            "gdla_set_wait_limit_ns": [ULL],
            "gdla_selftest_wait_timeout": [ULL, P, ctypes.POINTER(I)],
            "gdla_workspace_offset": [cfgp, I, I, I, I, ctypes.POINTER(SZ)],
            "gdla_status_string": [I],
            "gdla_set_stage_events": [ctypes.POINTER(P), I],
            "gdla_kernel_launches": [],
            "gdla_attn_prefill_noalloc": [cfgp, P, P, P, P, P, P, I, I, P],
            "gdla_prefill_varlen_fwd": [cfgp, wp, P, I, P, I, P, P, P, SZ, P],
            "gdla_decode_multi_fwd": [cfgp, abp, P, I, P, P, I, I, P, P, SZ, P],
            "gdla_latent_fwd": [cfgp, wp, P, I, I, P, P, SZ, P],
            "gdla_prefill_context_fwd": [cfgp, wp, P, I, I, P, I, P, P, P, SZ, P],
            "gdla_prefill_host_fwd": [cfgp, wp, P, I, I, P, I, P, SZ, P],
            "gdla_attn_train_workspace_size": [cfgp, I, I, ctypes.POINTER(SZ), ctypes.POINTER(SZ)],
            "gdla_attn_train_fwd": [cfgp, P, P, P, P, P, I, I, P, P, P, P, SZ, P],
            "gdla_attn_bwd": [cfgp, P, P, P, P, P, P, P, P, I, I, P, P, P, P, P, P, SZ, P],
            "gdla_quantize_latent_fp8": [cfgp, P, ctypes.c_longlong, P, P],
            "gdla_decode_fp8_fwd": [cfgp, abp, P, I, P, P, I, I, P, P, SZ, P],
            "gdla_dequantize_latent_fp8": [cfgp, P, ctypes.c_longlong, P, P],
        }
        for name, args in sig.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = {"gdla_status_string": ctypes.c_char_p,
                         "gdla_kernel_launches": ctypes.c_ulonglong}.get(name, I)
        _lib = L
    return _lib


def header_functions() -> list:
    """Names of the entry points declared in include/gdla.h."""
    src = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    return sorted(set(re.findall(r"\b(gdla_\w+)\s*\(", src)))


def _check(fn: str, rc: int) -> None:
    if rc != 0:
        raise GdlaError(fn, rc)


def _ptr(t, dtype=None, name="tensor"):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA tensor")
    return ctypes.c_void_p(t.data_ptr())


def _host_ptr(t, dtype, name):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous host (CPU) tensor")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def make_config(shape) -> gdla_config_t:
    """gdla_config_t from any object with the GdlaShape attribute names."""
    return gdla_config_t(shape.d_model, shape.q_rank, shape.kv_rank, shape.n_signal, shape.n_noise,
                         shape.n_kv_heads, shape.d_nope, shape.d_rope, shape.d_v, shape.window,
                         float(shape.rope_theta), float(shape.rms_eps))


def make_weights(w: dict, g_q=None, g_kv=None) -> gdla_weights_t:
    names = ("W_aQ", "W_bQ", "W_aKV", "W_bKV", "W_lambda", "W_G", "W_O")
    ptrs = [_ptr(w[n], torch.bfloat16, n) for n in names]
    return gdla_weights_t(*ptrs, _ptr(g_q, torch.bfloat16, "g_q"), _ptr(g_kv, torch.bfloat16, "g_kv"))


# ----------------------------------------------------------------------------- entry points
def gdla_status_string(status: int) -> str:
    return lib().gdla_status_string(status).decode()


def gdla_workspace_size(cfg: gdla_config_t, B: int, T: int, mode: int) -> int:
    out = ctypes.c_size_t(0)
    _check("gdla_workspace_size", lib().gdla_workspace_size(ctypes.byref(cfg), B, T, mode,
                                                            ctypes.byref(out)))
    return out.value


def gdla_workspace_offset(cfg: gdla_config_t, B: int, T: int, mode: int, which: int) -> int:
    out = ctypes.c_size_t(0)
    _check("gdla_workspace_offset", lib().gdla_workspace_offset(ctypes.byref(cfg), B, T, mode, which,
                                                                ctypes.byref(out)))
    return out.value


def gdla_absorbed_size(cfg: gdla_config_t) -> int:
    out = ctypes.c_size_t(0)
    _check("gdla_absorbed_size", lib().gdla_absorbed_size(ctypes.byref(cfg), ctypes.byref(out)))
    return out.value


def gdla_prefill_fwd(cfg, w: gdla_weights_t, x: torch.Tensor, y: torch.Tensor,
                     workspace: torch.Tensor, kv_cache_out: torch.Tensor | None = None,
                     cache_cap: int = 0, stream=None) -> None:
    B, T, _ = x.shape
    _check("gdla_prefill_fwd", lib().gdla_prefill_fwd(
        ctypes.byref(cfg), ctypes.byref(w), _ptr(x, torch.bfloat16, "x"), B, T,
        _ptr(y, torch.bfloat16, "y"), _ptr(kv_cache_out, torch.bfloat16, "kv_cache_out"),
        int(cache_cap), _ptr(workspace, None, "workspace"), workspace.numel() * workspace.element_size(),
        _stream(stream)))


def gdla_prefill_varlen_fwd(cfg, w: gdla_weights_t, x: torch.Tensor, cu_seqlens: torch.Tensor,
                            y: torch.Tensor, workspace: torch.Tensor,
                            kv_latent_out: torch.Tensor | None = None, stream=None) -> None:
    total = x.shape[0]
    _check("gdla_prefill_varlen_fwd", lib().gdla_prefill_varlen_fwd(
        ctypes.byref(cfg), ctypes.byref(w), _ptr(x, torch.bfloat16, "x"), total,
        _ptr(cu_seqlens, torch.int32, "cu_seqlens"), cu_seqlens.numel() - 1,
        _ptr(y, torch.bfloat16, "y"), _ptr(kv_latent_out, torch.bfloat16, "kv_latent_out"),
        _ptr(workspace, None, "workspace"), workspace.numel() * workspace.element_size(),
        _stream(stream)))


def gdla_prefill_host_fwd(cfg, w: gdla_weights_t, x_host: torch.Tensor, y_host: torch.Tensor,
                          workspace: torch.Tensor, n_pieces: int = 8, stream=None) -> None:
    """x_host, y_host: [B, T, d] bf16 CPU tensors (pin them for overlapped copies)."""
    B, T, _ = x_host.shape
    _check("gdla_prefill_host_fwd", lib().gdla_prefill_host_fwd(
        ctypes.byref(cfg), ctypes.byref(w), _host_ptr(x_host, torch.bfloat16, "x_host"), B, T,
        _host_ptr(y_host, torch.bfloat16, "y_host"), n_pieces, _ptr(workspace, None, "workspace"),
        workspace.numel() * workspace.element_size(), _stream(stream)))


def gdla_attn_train_workspace_size(cfg, B: int, T: int) -> tuple:
    f, b = ctypes.c_size_t(0), ctypes.c_size_t(0)
    _check("gdla_attn_train_workspace_size",
           lib().gdla_attn_train_workspace_size(ctypes.byref(cfg), B, T, ctypes.byref(f), ctypes.byref(b)))
    return f.value, b.value


def gdla_attn_train_fwd(cfg, qq, kv, kr16, lam, gate, B: int, T: int, dg_out, h_out, lse_out,
                        workspace, stream=None) -> None:
    _check("gdla_attn_train_fwd", lib().gdla_attn_train_fwd(
        ctypes.byref(cfg), _ptr(qq, torch.float16, "qq"), _ptr(kv, torch.float16, "kv"),
        _ptr(kr16, torch.float16, "kr16"), _ptr(lam, torch.float32, "lam"), _ptr(gate, torch.bfloat16, "gate"),
        B, T, _ptr(dg_out, torch.bfloat16, "dg_out"), _ptr(h_out, torch.bfloat16, "h_out"),
        _ptr(lse_out, torch.float32, "lse_out"), _ptr(workspace, None, "workspace"),
        workspace.numel() * workspace.element_size(), _stream(stream)))


def gdla_attn_bwd(cfg, qq, kv, kr16, lam, gate, h, lse, d_dg, B: int, T: int, d_qq, d_kv, d_kr,
                  d_lam, d_gate, workspace, stream=None) -> None:
    _check("gdla_attn_bwd", lib().gdla_attn_bwd(
        ctypes.byref(cfg), _ptr(qq, torch.float16, "qq"), _ptr(kv, torch.float16, "kv"),
        _ptr(kr16, torch.float16, "kr16"), _ptr(lam, torch.float32, "lam"), _ptr(gate, torch.bfloat16, "gate"),
        _ptr(h, torch.bfloat16, "h"), _ptr(lse, torch.float32, "lse"), _ptr(d_dg, torch.bfloat16, "d_dg"),
        B, T, _ptr(d_qq, torch.float32, "d_qq"), _ptr(d_kv, torch.float32, "d_kv"),
        _ptr(d_kr, torch.float32, "d_kr"), _ptr(d_lam, torch.float32, "d_lam"),
        _ptr(d_gate, torch.float32, "d_gate"), _ptr(workspace, None, "workspace"),
        workspace.numel() * workspace.element_size(), _stream(stream)))


def gdla_latent_fwd(cfg, w: gdla_weights_t, x: torch.Tensor, pos_offset: int, latent_out: torch.Tensor,
                    workspace: torch.Tensor, stream=None) -> None:
    T = x.shape[0]
    _check("gdla_latent_fwd", lib().gdla_latent_fwd(
        ctypes.byref(cfg), ctypes.byref(w), _ptr(x, torch.bfloat16, "x"), T, pos_offset,
        _ptr(latent_out, torch.bfloat16, "latent_out"), _ptr(workspace, None, "workspace"),
        workspace.numel() * workspace.element_size(), _stream(stream)))


FP8_ROW_BYTES = 608     # GDLA_FP8_ROW_BYTES


def gdla_quantize_latent_fp8(cfg, latent: torch.Tensor, out: torch.Tensor, stream=None) -> None:
    """bf16 latent rows [..., 576] -> MXFP8 rows [..., 608] (uint8), same leading shape."""
    rows = latent.numel() // (cfg.kv_rank + cfg.d_rope)
    if out.numel() != rows * FP8_ROW_BYTES:
        raise ValueError("out must hold rows x 608 bytes")
    _check("gdla_quantize_latent_fp8", lib().gdla_quantize_latent_fp8(
        ctypes.byref(cfg), _ptr(latent, torch.bfloat16, "latent"), rows, _ptr(out, torch.uint8, "out"),
        _stream(stream)))


def gdla_dequantize_latent_fp8(cfg, stored: torch.Tensor, out: torch.Tensor, stream=None) -> None:
    """MXFP8 rows [..., 608] (uint8) -> bf16 latent rows [..., 576]."""
    rows = stored.numel() // FP8_ROW_BYTES
    if out.numel() != rows * (cfg.kv_rank + cfg.d_rope):
        raise ValueError("out must hold rows x 576 values")
    _check("gdla_dequantize_latent_fp8", lib().gdla_dequantize_latent_fp8(
        ctypes.byref(cfg), _ptr(stored, torch.uint8, "stored"), rows, _ptr(out, torch.bfloat16, "out"),
        _stream(stream)))


def gdla_prefill_context_fwd(cfg, w: gdla_weights_t, x: torch.Tensor, pos_offset: int,
                             prefix_latent: torch.Tensor | None, y: torch.Tensor,
                             workspace: torch.Tensor, latent_out: torch.Tensor | None = None,
                             stream=None) -> None:
    T = x.shape[0]
    n_prefix = 0 if prefix_latent is None else prefix_latent.shape[0]
    _check("gdla_prefill_context_fwd", lib().gdla_prefill_context_fwd(
        ctypes.byref(cfg), ctypes.byref(w), _ptr(x, torch.bfloat16, "x"), T, pos_offset,
        _ptr(prefix_latent, torch.bfloat16, "prefix_latent") if n_prefix else None, n_prefix,
        _ptr(y, torch.bfloat16, "y"), _ptr(latent_out, torch.bfloat16, "latent_out"),
        _ptr(workspace, None, "workspace"), workspace.numel() * workspace.element_size(),
        _stream(stream)))


def gdla_absorb_weights(cfg, w: gdla_weights_t, dst: torch.Tensor, stream=None) -> gdla_absorbed_t:
    out = gdla_absorbed_t()
    _check("gdla_absorb_weights", lib().gdla_absorb_weights(
        ctypes.byref(cfg), ctypes.byref(w), _ptr(dst, None, "dst"), dst.numel() * dst.element_size(),
        ctypes.byref(out), _stream(stream)))
    return out


def gdla_decode_fwd(cfg, absorbed: gdla_absorbed_t, x_new: torch.Tensor, kv_cache: torch.Tensor,
                    cache_len: torch.Tensor, y: torch.Tensor, workspace: torch.Tensor,
                    stream=None) -> None:
    B = x_new.shape[0]
    cap = kv_cache.shape[1]
    _check("gdla_decode_fwd", lib().gdla_decode_fwd(
        ctypes.byref(cfg), ctypes.byref(absorbed), _ptr(x_new, torch.bfloat16, "x_new"),
        _ptr(kv_cache, torch.bfloat16, "kv_cache"), _ptr(cache_len, torch.int32, "cache_len"), cap, B,
        _ptr(y, torch.bfloat16, "y"), _ptr(workspace, None, "workspace"),
        workspace.numel() * workspace.element_size(), _stream(stream)))


def gdla_decode_multi_fwd(cfg, absorbed: gdla_absorbed_t, x_new: torch.Tensor, kv_cache: torch.Tensor,
                          cache_len: torch.Tensor, y: torch.Tensor, workspace: torch.Tensor,
                          stream=None) -> None:
    """x_new [n_seq, q_len, d]: q_len new tokens per sequence (positions cache_len + i)."""
    n_seq, q_len = x_new.shape[0], x_new.shape[1]
    _check("gdla_decode_multi_fwd", lib().gdla_decode_multi_fwd(
        ctypes.byref(cfg), ctypes.byref(absorbed), _ptr(x_new, torch.bfloat16, "x_new"), q_len,
        _ptr(kv_cache, torch.bfloat16, "kv_cache"), _ptr(cache_len, torch.int32, "cache_len"),
        kv_cache.shape[1], n_seq, _ptr(y, torch.bfloat16, "y"), _ptr(workspace, None, "workspace"),
        workspace.numel() * workspace.element_size(), _stream(stream)))


def gdla_decode_fp8_fwd(cfg, absorbed: gdla_absorbed_t, x_new: torch.Tensor, kv_cache8: torch.Tensor,
                        cache_len: torch.Tensor, y: torch.Tensor, workspace: torch.Tensor,
                        stream=None) -> None:
    """Decode over an MXFP8 cache kv_cache8 [n_seq, cap, 608] (uint8).  x_new [n_seq, d] (one new
    token per sequence) or [n_seq, q_len, d]; y has the shape of x_new."""
    n_seq = x_new.shape[0]
    q_len = x_new.shape[1] if x_new.dim() == 3 else 1
    _check("gdla_decode_fp8_fwd", lib().gdla_decode_fp8_fwd(
        ctypes.byref(cfg), ctypes.byref(absorbed), _ptr(x_new, torch.bfloat16, "x_new"), q_len,
        _ptr(kv_cache8, torch.uint8, "kv_cache8"), _ptr(cache_len, torch.int32, "cache_len"),
        kv_cache8.shape[1], n_seq, _ptr(y, torch.bfloat16, "y"), _ptr(workspace, None, "workspace"),
        workspace.numel() * workspace.element_size(), _stream(stream)))


def gdla_device_error(stream=None, clear: bool = True) -> int:
    site = ctypes.c_int(0)
    rc = lib().gdla_device_error(_stream(stream), ctypes.byref(site), int(clear))
    if rc not in (0, -5, -7):
        _check("gdla_device_error", rc)
    return site.value


def gdla_set_wait_limit_ns(ns: int) -> None:
    _check("gdla_set_wait_limit_ns", lib().gdla_set_wait_limit_ns(int(ns)))


def gdla_selftest_wait_timeout(limit_ns: int, stream=None) -> int:
    site = ctypes.c_int(0)
    rc = lib().gdla_selftest_wait_timeout(int(limit_ns), _stream(stream), ctypes.byref(site))
    if rc not in (0, -5, -7):
        _check("gdla_selftest_wait_timeout", rc)
    return site.value


def gdla_set_stage_events(events) -> None:
    """events: list of torch.cuda.Event (created with enable_timing=True), or [] to disable."""
    for e in events:            # torch creates the CUDA event on its first record
        if e.cuda_event == 0:
            e.record()
    arr = (ctypes.c_void_p * max(1, len(events)))(*[ctypes.c_void_p(e.cuda_event) for e in events])
    _check("gdla_set_stage_events", lib().gdla_set_stage_events(arr, len(events)))


def gdla_kernel_launches() -> int:
    return int(lib().gdla_kernel_launches())


def _header_define(name: str) -> int:
    m = re.search(r"#define\s+" + name + r"\s+(\d+)", open(HEADER).read())
    if not m:
        raise RuntimeError(f"{name} is not defined in {HEADER}")
    return int(m.group(1))


# token limit of gdla_attn_prefill_noalloc's fixed scratch, as the header defines it
GDLA_NOALLOC_MAX_TOKENS = _header_define("GDLA_NOALLOC_MAX_TOKENS")


def gdla_attn_prefill_noalloc(cfg, qq: torch.Tensor, kv: torch.Tensor, kr16: torch.Tensor,
                              lam: torch.Tensor, gate: torch.Tensor, dg: torch.Tensor, B: int, T: int,
                              stream=None) -> None:
    """Fused attention stage without a workspace (its scratch is a fixed array in the library)."""
    _check("gdla_attn_prefill_noalloc", lib().gdla_attn_prefill_noalloc(
        ctypes.byref(cfg), _ptr(qq, torch.float16, "qq"), _ptr(kv, torch.float16, "kv"),
        _ptr(kr16, torch.float16, "kr16"), _ptr(lam, torch.float32, "lam"),
        _ptr(gate, torch.bfloat16, "gate"), _ptr(dg, torch.bfloat16, "dg"), int(B), int(T),
        _stream(stream)))
