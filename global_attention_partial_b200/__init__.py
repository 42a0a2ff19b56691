"""Python binding of the MiMo-V2-Flash hybrid attention library (sm_100a).

Argument marshalling only: every function below passes torch tensors' device
pointers to the C ABI of include/mimo_attn.h (libmimo_attn.so, built in-tree
by global_attention_partial_b200/build.py) and returns its status. All
arithmetic runs in the library's CUDA kernels; there is no CPU fallback, and
importing the binding without the built library raises.

The layer follows "Add Xiaomi MiMo-V2" (huggingface/transformers PR 45144),
section "Additional useful info", and "feat(models): add Xiaomi MiMo v2
(mimo_v2_flash) text model support" (lablup/mlxcel issue 842), section
"Architecture, verified against upstream".
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmimo_attn.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_CUDA = range(5)
GLOBAL, SWA = 0, 1
BF16, FP32 = 0, 1
DEVERR_KV_LEN = 0x1
DEVERR_TIMEOUT = 0x2

EXPORTED = (
    "mimo_attn_rotary_dim",
    "mimo_attn_prefill_workspace_size",
    "mimo_attn_prefill",
    "mimo_attn_prefill_cached_workspace_size",
    "mimo_attn_prefill_cached",
    "mimo_attn_decode_workspace_size",
    "mimo_attn_decode",
    "mimo_attn_decode_static",
    "mimo_attn_qkv_project_workspace_size",
    "mimo_attn_qkv_project",
    "mimo_attn_decode_fp8kv_workspace_size",
    "mimo_attn_decode_fp8kv",
    "mimo_attn_quantize_fp8",
    "mimo_attn_get_device_error",
    "mimo_attn_status_string",
    "mimo_attn_debug_fail_launches",
    "mimo_attn_debug_set_wait_limit",
    "mimo_attn_debug_wait_probe",
    "mimo_attn_version",
)


class MimoAttnError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {status_string(status)} (status {status})")
        self.status = status


class mimo_attn_layer(ctypes.Structure):
    """Mirror of the C struct mimo_attn_layer."""
    _fields_ = [
        ("layer_type", ctypes.c_int32),
        ("num_q_heads", ctypes.c_int32),
        ("num_kv_heads", ctypes.c_int32),
        ("qk_dim", ctypes.c_int32),
        ("v_dim", ctypes.c_int32),
        ("rotary_dim", ctypes.c_int32),
        ("window", ctypes.c_int32),
        ("hidden_size", ctypes.c_int32),
        ("rope_theta", ctypes.c_double),
        ("softmax_scale", ctypes.c_float),
        ("sinks", ctypes.c_void_p),
    ]


_lib = None


def load() -> ctypes.CDLL:
    """Loads libmimo_attn.so; raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: run `python -m global_attention_partial_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    lp = ctypes.POINTER(mimo_attn_layer)
    lib.mimo_attn_rotary_dim.argtypes = [ctypes.c_double, i32]
    lib.mimo_attn_rotary_dim.restype = i32
    lib.mimo_attn_prefill_workspace_size.argtypes = [lp, i32, i32, i32]
    lib.mimo_attn_prefill_workspace_size.restype = sz
    lib.mimo_attn_prefill.argtypes = [lp, i32, i32, i32, vp, vp, vp, vp, vp, vp, vp, i32, vp, sz, vp]
    lib.mimo_attn_prefill.restype = i32
    lib.mimo_attn_prefill_cached_workspace_size.argtypes = [lp, i32, i32, i32, i32]
    lib.mimo_attn_prefill_cached_workspace_size.restype = sz
    lib.mimo_attn_prefill_cached.argtypes = [lp, i32, i32, i32, vp, vp, vp, vp, i32, vp, vp, vp, i32, vp, sz, vp]
    lib.mimo_attn_prefill_cached.restype = i32
    lib.mimo_attn_decode_workspace_size.argtypes = [lp, i32, i32, i32]
    lib.mimo_attn_decode_workspace_size.restype = sz
    lib.mimo_attn_decode.argtypes = [lp, i32, i32, vp, vp, vp, vp, vp, vp, i32, vp, vp, sz, vp]
    lib.mimo_attn_decode.restype = i32
    lib.mimo_attn_decode_static.argtypes = [lp, i32, i32, vp, vp, vp, vp, vp, vp, i32, vp, vp]
    lib.mimo_attn_decode_static.restype = i32
    f32 = ctypes.c_float
    lib.mimo_attn_qkv_project_workspace_size.argtypes = [lp, i32, i32, i32]
    lib.mimo_attn_qkv_project_workspace_size.restype = sz
    lib.mimo_attn_qkv_project.argtypes = [lp, i32, i32, vp, vp, vp, i32, vp, vp, vp, vp, vp, i32, vp, sz, vp]
    lib.mimo_attn_qkv_project.restype = i32
    lib.mimo_attn_decode_fp8kv_workspace_size.argtypes = [lp, i32, i32]
    lib.mimo_attn_decode_fp8kv_workspace_size.restype = sz
    lib.mimo_attn_decode_fp8kv.argtypes = [lp, i32, vp, vp, vp, vp, vp, vp, i32, f32, f32, vp, vp, sz, vp]
    lib.mimo_attn_decode_fp8kv.restype = i32
    lib.mimo_attn_quantize_fp8.argtypes = [vp, vp, sz, f32, vp]
    lib.mimo_attn_quantize_fp8.restype = i32
    lib.mimo_attn_get_device_error.argtypes = [ctypes.POINTER(ctypes.c_uint32)]
    lib.mimo_attn_get_device_error.restype = i32
    lib.mimo_attn_status_string.argtypes = [i32]
    lib.mimo_attn_status_string.restype = ctypes.c_char_p
    lib.mimo_attn_debug_fail_launches.argtypes = [i32]
    lib.mimo_attn_debug_fail_launches.restype = None
    lib.mimo_attn_debug_set_wait_limit.argtypes = [ctypes.c_longlong]
    lib.mimo_attn_debug_set_wait_limit.restype = i32
    lib.mimo_attn_debug_wait_probe.argtypes = [vp]
    lib.mimo_attn_debug_wait_probe.restype = i32
    lib.mimo_attn_version.argtypes = []
    lib.mimo_attn_version.restype = ctypes.c_char_p
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load().mimo_attn_status_string(int(status)).decode()


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if isinstance(t, torch.Tensor) and not t.is_cuda:
        # every pointer of the C ABI is a device pointer: a host address would
        # reach a kernel as a bad address
        raise ValueError("tensors passed to the library must be on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensors passed to the library must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def dtype_code(dtype: torch.dtype) -> int:
    if dtype == torch.bfloat16:
        return BF16
    if dtype == torch.float32:
        return FP32
    raise ValueError(f"unsupported dtype {dtype}")


def make_layer(layer_type: int, num_q_heads: int, num_kv_heads: int, qk_dim: int, v_dim: int,
               rotary_dim: int, window: int, rope_theta: float, hidden_size: int,
               sinks: Optional[torch.Tensor] = None, softmax_scale: float = 0.0) -> mimo_attn_layer:
    """Fills the C struct; `sinks` is a device fp32 tensor [Hq] or None (the
    struct keeps its pointer, so keep the tensor alive while the struct is used)."""
    if isinstance(sinks, torch.Tensor) and not (sinks.is_cuda and sinks.dtype == torch.float32 and sinks.is_contiguous()):
        raise ValueError("sinks must be a contiguous fp32 tensor on a CUDA device")
    return mimo_attn_layer(int(layer_type), int(num_q_heads), int(num_kv_heads), int(qk_dim),
                           int(v_dim), int(rotary_dim), int(window), int(hidden_size),
                           float(rope_theta), float(softmax_scale),
                           None if sinks is None else sinks.data_ptr())


def layer_from_config(pattern: Sequence[int], idx: int, *, num_attention_heads: int,
                      swa_num_key_value_heads: int, num_key_value_heads: int, head_dim: int,
                      v_head_dim: int, partial_rotary_factor: float, sliding_window_size: int,
                      rope_theta: float, swa_rope_theta: float, hidden_size: int,
                      sinks: Optional[torch.Tensor] = None) -> mimo_attn_layer:
    """Per-layer selection from the model config (lablup/mlxcel issue 842,
    "Architecture, verified against upstream"): pattern[idx] == 1 makes a
    sliding layer with swa_rope_theta, the sliding KV-head count, the window
    and the sink; otherwise a global layer with rope_theta, no window, no sink.
    The rotated width is int(partial_rotary_factor * head_dim)."""
    sliding = int(pattern[idx]) == 1
    rot = rotary_dim(partial_rotary_factor, head_dim)
    return make_layer(SWA if sliding else GLOBAL, num_attention_heads,
                      swa_num_key_value_heads if sliding else num_key_value_heads, head_dim,
                      v_head_dim, rot, sliding_window_size if sliding else 0,
                      swa_rope_theta if sliding else rope_theta, hidden_size,
                      sinks if sliding else None)


def rotary_dim(partial_rotary_factor: float, qk_dim: int) -> int:
    return int(load().mimo_attn_rotary_dim(float(partial_rotary_factor), int(qk_dim)))


def mimo_attn_prefill_workspace_size(layer: mimo_attn_layer, dtype: int, batch: int, seq: int) -> int:
    return int(load().mimo_attn_prefill_workspace_size(ctypes.byref(layer), dtype, batch, seq))


def mimo_attn_decode_workspace_size(layer: mimo_attn_layer, dtype: int, batch: int, cache_capacity: int) -> int:
    return int(load().mimo_attn_decode_workspace_size(ctypes.byref(layer), dtype, batch, cache_capacity))


def mimo_attn_prefill(layer: mimo_attn_layer, dtype: int, batch: int, seq: int, q, k, v, positions, out,
                      k_cache=None, v_cache=None, cache_capacity: int = 0, workspace=None,
                      workspace_bytes: int = 0, stream=None) -> int:
    """Same arguments as the C entry point; tensors in place of pointers."""
    return int(load().mimo_attn_prefill(
        ctypes.byref(layer), dtype, batch, seq, _ptr(q), _ptr(k), _ptr(v), _ptr(positions), _ptr(out),
        _ptr(k_cache), _ptr(v_cache), int(cache_capacity), _ptr(workspace), int(workspace_bytes),
        _stream(stream)))


def mimo_attn_prefill_cached_workspace_size(layer: mimo_attn_layer, dtype: int, batch: int, seq: int,
                                            max_past_len: int) -> int:
    return int(load().mimo_attn_prefill_cached_workspace_size(ctypes.byref(layer), dtype, batch, seq,
                                                              int(max_past_len)))


def mimo_attn_prefill_cached(layer: mimo_attn_layer, dtype: int, batch: int, seq: int, q, k, v, past_lens,
                             max_past_len: int, out, k_cache, v_cache, cache_capacity: int, workspace=None,
                             workspace_bytes: int = 0, stream=None) -> int:
    """Same arguments as the C entry point; tensors in place of pointers."""
    return int(load().mimo_attn_prefill_cached(
        ctypes.byref(layer), dtype, batch, seq, _ptr(q), _ptr(k), _ptr(v), _ptr(past_lens), int(max_past_len),
        _ptr(out), _ptr(k_cache), _ptr(v_cache), int(cache_capacity), _ptr(workspace), int(workspace_bytes),
        _stream(stream)))


def mimo_attn_decode(layer: mimo_attn_layer, dtype: int, batch: int, q, k_new, v_new, kv_lens, k_cache,
                     v_cache, cache_capacity: int, out, workspace=None, workspace_bytes: int = 0,
                     stream=None) -> int:
    """Same arguments as the C entry point; tensors in place of pointers."""
    return int(load().mimo_attn_decode(
        ctypes.byref(layer), dtype, batch, _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(kv_lens),
        _ptr(k_cache), _ptr(v_cache), int(cache_capacity), _ptr(out), _ptr(workspace),
        int(workspace_bytes), _stream(stream)))


def mimo_attn_decode_static(layer: mimo_attn_layer, dtype: int, batch: int, q, k_new, v_new, kv_lens, k_cache,
                            v_cache, cache_capacity: int, out, stream=None) -> int:
    """Decode with no allocation at all: the split partials live in the
    library's built-in 16 MiB scratch (see include/mimo_attn.h). For callers
    that cannot allocate device memory; concurrent calls race on the scratch."""
    return int(load().mimo_attn_decode_static(
        ctypes.byref(layer), dtype, batch, _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(kv_lens),
        _ptr(k_cache), _ptr(v_cache), int(cache_capacity), _ptr(out), _stream(stream)))


def mimo_attn_qkv_project_workspace_size(layer: mimo_attn_layer, batch: int, seq: int, max_past_len: int) -> int:
    return int(load().mimo_attn_qkv_project_workspace_size(ctypes.byref(layer), batch, seq, int(max_past_len)))


def mimo_attn_qkv_project(layer: mimo_attn_layer, batch: int, seq: int, x, w_qkv, past_lens, max_past_len: int,
                          q_out, k_out, v_out, k_cache, v_cache, cache_capacity: int, workspace=None,
                          workspace_bytes: int = 0, stream=None) -> int:
    """Same arguments as the C entry point; tensors (or None) in place of pointers."""
    return int(load().mimo_attn_qkv_project(
        ctypes.byref(layer), batch, seq, _ptr(x), _ptr(w_qkv), _ptr(past_lens), int(max_past_len), _ptr(q_out),
        _ptr(k_out), _ptr(v_out), _ptr(k_cache), _ptr(v_cache), int(cache_capacity), _ptr(workspace),
        int(workspace_bytes), _stream(stream)))


def mimo_attn_decode_fp8kv_workspace_size(layer: mimo_attn_layer, batch: int, cache_capacity: int) -> int:
    return int(load().mimo_attn_decode_fp8kv_workspace_size(ctypes.byref(layer), batch, cache_capacity))


def mimo_attn_decode_fp8kv(layer: mimo_attn_layer, batch: int, q, k_new, v_new, kv_lens, k_cache, v_cache,
                           cache_capacity: int, k_scale: float, v_scale: float, out, workspace=None,
                           workspace_bytes: int = 0, stream=None) -> int:
    """Same arguments as the C entry point; tensors in place of pointers
    (k_cache / v_cache uint8 E4M3 codes)."""
    return int(load().mimo_attn_decode_fp8kv(
        ctypes.byref(layer), batch, _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(kv_lens), _ptr(k_cache),
        _ptr(v_cache), int(cache_capacity), float(k_scale), float(v_scale), _ptr(out), _ptr(workspace),
        int(workspace_bytes), _stream(stream)))


def mimo_attn_quantize_fp8(src, dst, n: int, scale: float, stream=None) -> int:
    return int(load().mimo_attn_quantize_fp8(_ptr(src), _ptr(dst), int(n), float(scale), _stream(stream)))


def mimo_attn_get_device_error() -> int:
    bits = ctypes.c_uint32(0)
    st = load().mimo_attn_get_device_error(ctypes.byref(bits))
    if st != OK:
        raise MimoAttnError(st, "mimo_attn_get_device_error")
    return int(bits.value)


def mimo_attn_debug_fail_launches(enable: bool) -> None:
    load().mimo_attn_debug_fail_launches(1 if enable else 0)


def mimo_attn_debug_set_wait_limit(cycles: int) -> int:
    return load().mimo_attn_debug_set_wait_limit(int(cycles))


def mimo_attn_debug_wait_probe(stream=None) -> int:
    return load().mimo_attn_debug_wait_probe(_stream(stream))


def version() -> str:
    return load().mimo_attn_version().decode()


# ------------------------------------------------------------ conveniences
def _check(status: int, what: str):
    if status != OK:
        raise MimoAttnError(status, what)


def prefill(layer: mimo_attn_layer, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
            positions: Optional[torch.Tensor] = None, k_cache=None, v_cache=None,
            out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
            stream=None) -> torch.Tensor:
    """Runs mimo_attn_prefill; allocates `out` and the workspace with torch when
    not given. q [B,S,Hq,Dqk], k [B,S,Hkv,Dqk], v [B,S,Hkv,Dv] on the GPU."""
    B, S = q.shape[0], q.shape[1]
    dt = dtype_code(q.dtype)
    if out is None:
        out = torch.empty((B, S, layer.num_q_heads, layer.v_dim), dtype=q.dtype, device=q.device)
    need = mimo_attn_prefill_workspace_size(layer, dt, B, S)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    cap = 0 if k_cache is None else k_cache.shape[1]
    _check(mimo_attn_prefill(layer, dt, B, S, q, k, v, positions, out, k_cache, v_cache, cap, workspace,
                             0 if workspace is None else workspace.numel(), stream), "mimo_attn_prefill")
    return out


def prefill_cached(layer: mimo_attn_layer, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                   past_lens: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                   max_past_len: Optional[int] = None, out: Optional[torch.Tensor] = None,
                   workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Runs mimo_attn_prefill_cached (a chunk after past_lens[b] cached tokens;
    updates the caches in place). max_past_len defaults to max(past_lens), read
    on the host (one synchronisation); pass it to avoid that."""
    B, S = q.shape[0], q.shape[1]
    dt = dtype_code(q.dtype)
    if max_past_len is None:
        max_past_len = int(past_lens.max().item()) if past_lens.numel() else 0
    if out is None:
        out = torch.empty((B, S, layer.num_q_heads, layer.v_dim), dtype=q.dtype, device=q.device)
    need = mimo_attn_prefill_cached_workspace_size(layer, dt, B, S, max_past_len)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    _check(mimo_attn_prefill_cached(layer, dt, B, S, q, k, v, past_lens, max_past_len, out, k_cache, v_cache,
                                    k_cache.shape[1], workspace, 0 if workspace is None else workspace.numel(),
                                    stream), "mimo_attn_prefill_cached")
    return out


def decode(layer: mimo_attn_layer, q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor,
           kv_lens: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
           out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
           stream=None) -> torch.Tensor:
    """Runs mimo_attn_decode (updates the caches in place)."""
    B = q.shape[0]
    dt = dtype_code(q.dtype)
    cap = k_cache.shape[1]
    if out is None:
        out = torch.empty((B, layer.num_q_heads, layer.v_dim), dtype=q.dtype, device=q.device)
    need = mimo_attn_decode_workspace_size(layer, dt, B, cap)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    _check(mimo_attn_decode(layer, dt, B, q, k_new, v_new, kv_lens, k_cache, v_cache, cap, out, workspace,
                            0 if workspace is None else workspace.numel(), stream), "mimo_attn_decode")
    return out


def decode_fp8kv(layer: mimo_attn_layer, q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor,
                 kv_lens: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, k_scale: float,
                 v_scale: float, out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                 stream=None) -> torch.Tensor:
    """Runs mimo_attn_decode_fp8kv: bf16 q/k_new/v_new, uint8 E4M3 caches
    (updated in place), bf16 out."""
    B = q.shape[0]
    cap = k_cache.shape[1]
    if k_cache.dtype != torch.uint8 or v_cache.dtype != torch.uint8:
        raise ValueError("fp8 caches are uint8 tensors of E4M3 codes")
    if out is None:
        out = torch.empty((B, layer.num_q_heads, layer.v_dim), dtype=q.dtype, device=q.device)
    need = mimo_attn_decode_fp8kv_workspace_size(layer, B, cap)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    _check(mimo_attn_decode_fp8kv(layer, B, q, k_new, v_new, kv_lens, k_cache, v_cache, cap, k_scale, v_scale,
                                  out, workspace, 0 if workspace is None else workspace.numel(), stream),
           "mimo_attn_decode_fp8kv")
    return out


def quantize_fp8(src: torch.Tensor, scale: float, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """E4M3 codes of src / scale (src bf16 on the GPU), same shape, uint8."""
    if src.dtype != torch.bfloat16:
        raise ValueError("quantize_fp8 takes bf16")
    if out is None:
        out = torch.empty(src.shape, dtype=torch.uint8, device=src.device)
    _check(mimo_attn_quantize_fp8(src, out, src.numel(), scale, stream), "mimo_attn_quantize_fp8")
    return out


def qkv_project(layer: mimo_attn_layer, x: torch.Tensor, w_qkv: torch.Tensor, past_lens: Optional[torch.Tensor] = None,
                max_past_len: Optional[int] = None, k_cache: Optional[torch.Tensor] = None,
                v_cache: Optional[torch.Tensor] = None, want_kv: bool = True, stream=None):
    """Runs mimo_attn_qkv_project on x [B, S, hidden]: returns (q, k, v) with q
    and k rotated ([B, S, H, D]; k and v are None when want_kv is False) and
    fills the caches when given. max_past_len defaults to max(past_lens), read
    on the host."""
    B, S = x.shape[0], x.shape[1]
    if max_past_len is None:
        max_past_len = int(past_lens.max().item()) if past_lens is not None and past_lens.numel() else 0
    q = torch.empty((B, S, layer.num_q_heads, layer.qk_dim), dtype=x.dtype, device=x.device)
    k = v = None
    if want_kv:
        k = torch.empty((B, S, layer.num_kv_heads, layer.qk_dim), dtype=x.dtype, device=x.device)
        v = torch.empty((B, S, layer.num_kv_heads, layer.v_dim), dtype=x.dtype, device=x.device)
    need = mimo_attn_qkv_project_workspace_size(layer, B, S, max_past_len)
    ws = torch.empty(max(need, 256), dtype=torch.uint8, device=x.device)
    cap = 0 if k_cache is None else k_cache.shape[1]
    _check(mimo_attn_qkv_project(layer, B, S, x, w_qkv, past_lens, max_past_len, q, k, v, k_cache, v_cache, cap,
                                 ws, ws.numel(), stream), "mimo_attn_qkv_project")
    return q, k, v
