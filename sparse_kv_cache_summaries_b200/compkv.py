"""Thin Python binding of libcompkv.so (the C ABI in include/compkv.h).

Argument marshalling only: every step of the decode path runs in the library's CUDA kernels.
Tensors are PyTorch CUDA tensors (PyTorch provides device memory and streams); each call passes
their device pointers and the current CUDA stream to the C function of the same name
(``compkv_<name>``) and raises ``CompKVError`` on a non-zero status. There is no fallback: if
the library is missing or fails to load, every call raises.
"""
from __future__ import annotations

import ctypes
import dataclasses
import pathlib
import re

import torch

LIB_PATH = pathlib.Path(__file__).resolve().with_name("libcompkv.so")
HEADER = pathlib.Path(__file__).resolve().parent.parent / "include" / "compkv.h"

MODES = {"compkv": 0, "mass": 1, "mass_comp": 2}
SUMMARY_DTYPES = {"fp32": 0, "fp16": 1}
_DTYPES = {torch.bfloat16: 0, torch.float32: 1}
BLOCK_SIZE = 16


class CompKVError(RuntimeError):
    def __init__(self, status: int, where: str):
        msg = f"{where}: {status_string(status)} ({status})"
        if status == -5:
            msg += f": {last_cuda_error()}"
        super().__init__(msg)
        self.status = status


class Shape(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("n_q_heads", ctypes.c_int32),
                ("n_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("ctx_len", ctypes.c_int32), ("block_size", ctypes.c_int32),
                ("n_groups", ctypes.c_int32), ("summary_dtype", ctypes.c_int32)]


@dataclasses.dataclass(frozen=True)
class LayerShape:
    """Problem shape of one attention layer (mirrors compkv_shape)."""
    batch: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    ctx_len: int
    n_groups: int = 4
    block_size: int = BLOCK_SIZE
    summary_dtype: str = "fp32"  # storage of mean_k / mean_v: "fp32" or "fp16"

    @property
    def n_blocks(self) -> int:
        return -(-self.ctx_len // self.block_size)

    @property
    def group_size(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    def c(self) -> Shape:
        return Shape(self.batch, self.n_q_heads, self.n_kv_heads, self.head_dim, self.ctx_len,
                     self.block_size, self.n_groups, SUMMARY_DTYPES[self.summary_dtype])


_lib = None


def lib() -> ctypes.CDLL:
    """Load libcompkv.so once; raise if it is not built."""
    global _lib
    if _lib is None:
        if not LIB_PATH.exists():
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m sparse_kv_cache_summaries_b200.build`")
        L = ctypes.CDLL(str(LIB_PATH))
        P, I32, SZ, F = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t, ctypes.c_float
        SP = ctypes.POINTER(Shape)
        sig = {
            "compkv_num_selected": (I32, [SP, I32]),
            "compkv_workspace_bytes": (SZ, [SP, I32]),
            "compkv_full_workspace_bytes": (SZ, [SP]),
            "compkv_build_summaries": (ctypes.c_int, [SP, ctypes.c_int, P, P, P, P, P, P, P, P]),
            "compkv_append": (ctypes.c_int, [SP, ctypes.c_int, P, P, P, P, P, P, P, P, P, P, P]),
            "compkv_score_select": (ctypes.c_int, [SP, ctypes.c_int, ctypes.c_int, P, P, P, P, P,
                                                   I32, F, P, P, P, SZ, P]),
            "compkv_score_stream": (ctypes.c_int, [SP, ctypes.c_int, ctypes.c_int, P, P, P, P, P,
                                                   I32, F, P, SZ, P]),
            "compkv_sparse_decode": (ctypes.c_int, [SP, ctypes.c_int, ctypes.c_int, P, P, P, P,
                                                    P, P, P, I32, F, P, P, SZ, P]),
            "compkv_decode_step": (ctypes.c_int, [SP, ctypes.c_int, ctypes.c_int, P, P, P, P, P,
                                                  P, P, I32, F, P, P, P, P, SZ, P]),
            "compkv_full_decode": (ctypes.c_int, [SP, ctypes.c_int, P, P, P, P, F, P, P, SZ, P]),
            "compkv_decode_step_static": (ctypes.c_int, [SP, ctypes.c_int, ctypes.c_int, P, P, P,
                                                         P, P, P, P, I32, F, P, P, P, P]),
            "compkv_read_device_status": (ctypes.c_int, [P, P, ctypes.POINTER(I32)]),
            "compkv_static_read_device_status": (ctypes.c_int, [P, ctypes.POINTER(I32)]),
            "compkv_status_string": (ctypes.c_char_p, [ctypes.c_int]),
            "compkv_last_cuda_error": (ctypes.c_char_p, []),
            "compkv_version": (ctypes.c_int, []),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype, fn.argtypes = res, args
        _lib = L
    return _lib


def header_functions() -> list[str]:
    """Names of the functions include/compkv.h declares."""
    text = HEADER.read_text()
    return sorted(set(re.findall(r"\b(compkv_\w+)\s*\(", text)))


def _p(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dt(t: torch.Tensor) -> int:
    if t.dtype not in _DTYPES:
        raise TypeError(f"unsupported dtype {t.dtype}")
    return _DTYPES[t.dtype]


def _ok(status: int, where: str) -> None:
    if status != 0:
        raise CompKVError(status, where)


def status_string(status: int) -> str:
    return lib().compkv_status_string(status).decode()


def last_cuda_error() -> str:
    return lib().compkv_last_cuda_error().decode()


def version() -> int:
    return lib().compkv_version()


def num_selected(shape: LayerShape, budget_tokens: int) -> int:
    k = lib().compkv_num_selected(ctypes.byref(shape.c()), budget_tokens)
    _ok(min(k, 0), "num_selected")
    return k


def workspace_bytes(shape: LayerShape, budget_tokens: int) -> int:
    return lib().compkv_workspace_bytes(ctypes.byref(shape.c()), budget_tokens)


def full_workspace_bytes(shape: LayerShape) -> int:
    return lib().compkv_full_workspace_bytes(ctypes.byref(shape.c()))


# ------------------------------------------------------------------ buffers (torch allocations)

@dataclasses.dataclass
class Summaries:
    mean_k: torch.Tensor   # [B, Hkv, Nb, d] fp32 or fp16 (LayerShape.summary_dtype)
    var_g: torch.Tensor    # [B, Hkv, Nb, r] fp32
    mean_v: torch.Tensor   # [B, Hkv, Nb, d] fp32 or fp16
    count: torch.Tensor    # [B, Hkv, Nb] int32


def empty_summaries(shape: LayerShape, device="cuda") -> Summaries:
    B, H, nb, d, r = shape.batch, shape.n_kv_heads, shape.n_blocks, shape.head_dim, shape.n_groups
    f = dict(device=device, dtype=torch.float32)
    m = dict(device=device, dtype=torch.float16 if shape.summary_dtype == "fp16" else torch.float32)
    return Summaries(torch.empty((B, H, nb, d), **m), torch.empty((B, H, nb, r), **f),
                     torch.empty((B, H, nb, d), **m),
                     torch.empty((B, H, nb), device=device, dtype=torch.int32))


def new_workspace(shape: LayerShape, budget_tokens: int, device="cuda") -> torch.Tensor:
    """Zero-filled workspace for the sparse step (the library needs it zeroed once)."""
    return torch.zeros(workspace_bytes(shape, budget_tokens), dtype=torch.uint8, device=device)


def new_full_workspace(shape: LayerShape, device="cuda") -> torch.Tensor:
    return torch.zeros(full_workspace_bytes(shape), dtype=torch.uint8, device=device)


# ------------------------------------------------------------------ calls

def build_summaries(shape: LayerShape, K: torch.Tensor, V: torch.Tensor, out: Summaries,
                    ctx_lens: torch.Tensor | None = None, stream=None) -> Summaries:
    _ok(lib().compkv_build_summaries(ctypes.byref(shape.c()), _dt(K), _p(K), _p(V), _p(ctx_lens),
                                     _p(out.mean_k), _p(out.var_g), _p(out.mean_v), _p(out.count),
                                     _stream(stream)), "build_summaries")
    return out


def append(shape: LayerShape, k_new: torch.Tensor, v_new: torch.Tensor, positions: torch.Tensor,
           summ: Summaries, K: torch.Tensor | None = None, V: torch.Tensor | None = None,
           status: torch.Tensor | None = None, stream=None) -> Summaries:
    """One new token per sequence enters the cache: updates `summ` in place (and stores the token
    at row positions[b] of K/V when given). positions: int32 [B] on the device."""
    _ok(lib().compkv_append(ctypes.byref(shape.c()), _dt(k_new), _p(k_new), _p(v_new),
                            _p(positions), _p(K), _p(V), _p(summ.mean_k), _p(summ.var_g),
                            _p(summ.mean_v), _p(summ.count), _p(status), _stream(stream)),
        "append")
    return summ


def score_select(shape: LayerShape, q: torch.Tensor, summ: Summaries, budget_tokens: int,
                 sel_idx: torch.Tensor, workspace: torch.Tensor, mode: str = "compkv",
                 scores: torch.Tensor | None = None, softmax_scale: float = 0.0,
                 stream=None) -> torch.Tensor:
    _ok(lib().compkv_score_select(ctypes.byref(shape.c()), _dt(q), MODES[mode], _p(q),
                                  _p(summ.mean_k), _p(summ.var_g), _p(summ.mean_v),
                                  _p(summ.count), budget_tokens, softmax_scale, _p(sel_idx),
                                  _p(scores), _p(workspace), workspace.numel(), _stream(stream)),
        "score_select")
    return sel_idx


def score_stream(shape: LayerShape, q: torch.Tensor, summ: Summaries, budget_tokens: int,
                 workspace: torch.Tensor, mode: str = "compkv", softmax_scale: float = 0.0,
                 stream=None) -> None:
    """The streaming pass of score_select alone (its outputs stay in the workspace)."""
    _ok(lib().compkv_score_stream(ctypes.byref(shape.c()), _dt(q), MODES[mode], _p(q),
                                  _p(summ.mean_k), _p(summ.var_g), _p(summ.mean_v),
                                  _p(summ.count), budget_tokens, softmax_scale, _p(workspace),
                                  workspace.numel(), _stream(stream)), "score_stream")


def sparse_decode(shape: LayerShape, q: torch.Tensor, K: torch.Tensor, V: torch.Tensor,
                  summ: Summaries, sel_idx: torch.Tensor, budget_tokens: int, out: torch.Tensor,
                  workspace: torch.Tensor, mode: str = "compkv", softmax_scale: float = 0.0,
                  stream=None) -> torch.Tensor:
    _ok(lib().compkv_sparse_decode(ctypes.byref(shape.c()), _dt(q), MODES[mode], _p(q), _p(K),
                                   _p(V), _p(summ.mean_k), _p(summ.mean_v), _p(summ.count),
                                   _p(sel_idx), budget_tokens, softmax_scale, _p(out),
                                   _p(workspace), workspace.numel(), _stream(stream)),
        "sparse_decode")
    return out


def decode_step(shape: LayerShape, q: torch.Tensor, K: torch.Tensor, V: torch.Tensor,
                summ: Summaries, budget_tokens: int, sel_idx: torch.Tensor, out: torch.Tensor,
                workspace: torch.Tensor, mode: str = "compkv", scores: torch.Tensor | None = None,
                softmax_scale: float = 0.0, stream=None) -> torch.Tensor:
    _ok(lib().compkv_decode_step(ctypes.byref(shape.c()), _dt(q), MODES[mode], _p(q), _p(K),
                                 _p(V), _p(summ.mean_k), _p(summ.var_g), _p(summ.mean_v),
                                 _p(summ.count), budget_tokens, softmax_scale, _p(sel_idx),
                                 _p(scores), _p(out), _p(workspace), workspace.numel(),
                                 _stream(stream)), "decode_step")
    return out


def decode_step_static(shape: LayerShape, q: torch.Tensor, K: torch.Tensor, V: torch.Tensor,
                       summ: Summaries, budget_tokens: int, sel_idx: torch.Tensor,
                       out: torch.Tensor, mode: str = "compkv", scores: torch.Tensor | None = None,
                       softmax_scale: float = 0.0, stream=None) -> torch.Tensor:
    """decode_step without a workspace: the library's own static device scratch is used (for
    callers that cannot allocate device memory; see compkv_decode_step_static)."""
    _ok(lib().compkv_decode_step_static(ctypes.byref(shape.c()), _dt(q), MODES[mode], _p(q),
                                        _p(K), _p(V), _p(summ.mean_k), _p(summ.var_g),
                                        _p(summ.mean_v), _p(summ.count), budget_tokens,
                                        softmax_scale, _p(sel_idx), _p(scores), _p(out),
                                        _stream(stream)), "decode_step_static")
    return out


def full_decode(shape: LayerShape, q: torch.Tensor, K: torch.Tensor, V: torch.Tensor,
                out: torch.Tensor, workspace: torch.Tensor, ctx_lens: torch.Tensor | None = None,
                softmax_scale: float = 0.0, stream=None) -> torch.Tensor:
    _ok(lib().compkv_full_decode(ctypes.byref(shape.c()), _dt(q), _p(q), _p(K), _p(V),
                                 _p(ctx_lens), softmax_scale, _p(out), _p(workspace),
                                 workspace.numel(), _stream(stream)), "full_decode")
    return out


def read_device_status(workspace: torch.Tensor, stream=None) -> int:
    st = ctypes.c_int32(0)
    _ok(lib().compkv_read_device_status(_p(workspace), _stream(stream), ctypes.byref(st)),
        "read_device_status")
    return st.value


def static_read_device_status(stream=None) -> int:
    """Status word of the scratch array that decode_step_static uses (read and cleared)."""
    st = ctypes.c_int32(0)
    _ok(lib().compkv_static_read_device_status(_stream(stream), ctypes.byref(st)),
        "static_read_device_status")
    return st.value
