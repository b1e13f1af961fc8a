"""ctypes binding of libtokengate.so (argument marshalling only).

Every computation runs in the CUDA library; this module checks tensor
types, shapes and devices, passes raw pointers and the current CUDA stream,
and turns a non-zero tg_status into an exception.  There is no CPU fallback:
when the library is missing, loading fails loudly.
"""

from __future__ import annotations

import ctypes as C
import os
import threading

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtokengate.so")
_lock = threading.Lock()
_lib = None

TG_OK, TG_ERR_INVALID_ARG, TG_ERR_UNSUPPORTED, TG_ERR_CUDA, TG_ERR_TIMEOUT = range(5)
_STATUS = {1: "TG_ERR_INVALID_ARG", 2: "TG_ERR_UNSUPPORTED", 3: "TG_ERR_CUDA", 4: "TG_ERR_TIMEOUT"}

P = C.c_void_p
i32, i64, f32 = C.c_int, C.c_int64, C.c_float


class TokenGateError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{_STATUS.get(status, status)}: {msg}")
        self.status = status


class PrefillLayerArgs(C.Structure):
    _fields_ = [
        ("hidden", P), ("cu_seqlens", P), ("span", P), ("k", P), ("B", i32), ("T", i64), ("D", i32),
        ("Wg", P), ("b1", P), ("w2", P), ("b2", f32), ("I", i32), ("eps", f32),
        ("cu_kept", P), ("M_total", i64), ("max_M", i32),
        ("scores", P), ("keep", P), ("hidden_kept", P), ("pos", P), ("rank", P), ("gls", P), ("kept_idx", P),
        ("n_layers", i32), ("Hq", i32), ("Hkv", i32), ("d", i32), ("sm_scale", f32),
        ("q", P), ("kk", P), ("v", P), ("g", P), ("c", P), ("out", P), ("lse", P),
        ("attn_ws", P), ("attn_ws_bytes", C.c_size_t),
        ("n_gather", C.c_int), ("gather_src", C.POINTER(P)), ("gather_dst", C.POINTER(P)),
        ("gather_row_bytes", C.POINTER(C.c_int64)),
    ]


# the C ABI's exported symbols and their argument types
SIGNATURES = {
    "tg_abi_version": ([], i32),
    "tg_last_error_string": ([], C.c_char_p),
    "tg_kept_count": ([P, P, P, i32, P], i64),
    "tg_gate_prepare": ([P, P, i32, i32, P, P], i32),
    "tg_score": ([P, P, P, i32, i64, i32, P, P, P, f32, i32, f32, P, P], i32),
    "tg_select_topk": ([P, P, P, P, i32, i64, P, P, P, P, P, P, P], i32),
    "tg_compact": ([P, P, P, P, P, i32, i64, i32, P, i64, P, P, P, P, P, P], i32),
    "tg_gated_attention": ([P, P, P, P, i32, i64, i32, i32, i32, i32, P, P, P, P, P, f32, P, P, P, C.c_size_t, P],
                           i32),
    "tg_gated_attention_gates": ([P, P, P, P, i32, i64, i32, i32, i32, i32, P, P, i32, P, P, P, f32, P, P, P,
                                  C.c_size_t, P], i32),
    "tg_next_gate_span": ([P, P, i32, P], i32),
    "tg_gated_attention_backward_workspace_size": ([i64, i32, i32, i32], C.c_size_t),
    "tg_gated_attention_backward": ([P, P, P, P, P, P, P, i32, i64, i32, i32, i32, i32, P, P, P, P, P, f32,
                                     P, P, P, P, P, P, P, P, C.c_size_t, P], i32),
    "tg_gated_attention_backward_gates": ([P, P, P, P, P, P, P, i32, i64, i32, i32, i32, i32, P, P, i32, P, P, P,
                                           f32, P, P, P, P, P, P, P, P, C.c_size_t, P], i32),
    "tg_gated_attention_workspace_size": ([i32, i32, i32, i32, i32], C.c_size_t),
    "tg_gated_prefill_workspace_size": ([i32, i32, i32, i32, i32, i32], C.c_size_t),
    "tg_gated_attention_noalloc": ([P, P, P, P, i32, i64, i32, i32, i32, i32, P, P, P, P, P, f32, P, P, P], i32),
    "tg_gated_prefill_layer": ([C.POINTER(PrefillLayerArgs), P], i32),
    "tg_gather_rows": ([P, i64, i64, P, i64, P, P], i32),
    "tg_masked_gated_attention_workspace_size": ([i32, i64, i64, i32, i32, i32, i32], C.c_size_t),
    "tg_masked_gated_attention": ([P, P, P, P, P, P, P, P, i32, i64, i64, i32, i32, i32, i32, P, P, f32, P, P, P,
                                   C.c_size_t, P], i32),
    "tg_device_status": ([P, i32, P], i32),
    "tg_selftest_bounded_wait": ([i64, P], i32),
    "tg_selftest_exp2": ([P, P, i64, P], i32),
}


def load():
    """Load libtokengate.so (raises when it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise ImportError(
                    f"{LIB_PATH} is missing: build it with `python -m learned_token_pruning_rmsnorm_b200.build`")
            lib = C.CDLL(LIB_PATH)
            for name, (args, res) in SIGNATURES.items():
                fn = getattr(lib, name)
                fn.argtypes = args
                fn.restype = res
            _lib = lib
    return _lib


def check(status: int) -> None:
    if status != TG_OK:
        msg = load().tg_last_error_string()
        raise TokenGateError(status, msg.decode() if msg else "")


def ptr(t) -> int | None:
    if t is None:
        return None
    return t.data_ptr()


def stream_handle(device=None) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def host_i32(a) -> np.ndarray:
    if isinstance(a, torch.Tensor):
        a = a.detach().cpu().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))
