"""Python binding of libtpblock (ctypes): the C-ABI calls under the same names.

Argument marshalling only: tensors are passed as device pointers with the current torch CUDA
stream; every step of the block runs in the library's CUDA kernels.  There is no fallback: if the
library is missing or a call fails, a ``TpError`` is raised.  The C declarations, layouts and
error behaviour are documented in ``include/tp_block.h``.
"""

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# TPBLOCK_LIBRARY may point at another build of the same library (e.g. a tuning variant)
LIB_PATH = os.environ.get("TPBLOCK_LIBRARY") or os.path.join(_HERE, "libtpblock.so")

TP_OK, TP_ERR_INVALID_ARG, TP_ERR_SHAPE, TP_ERR_UNSUPPORTED, TP_ERR_WORKSPACE, TP_ERR_CUDA, \
    TP_ERR_TIMEOUT = range(7)
TP_F32, TP_BF16 = 0, 1
ACT = {"identity": 0, "relu": 1, "gelu": 2, "swiglu": 3}
DTYPE = {"f32": TP_F32, "bf16": TP_BF16}
TORCH_OF = {TP_F32: torch.float32, TP_BF16: torch.bfloat16}
TP_REDUCE_SEPARATE, TP_REDUCE_FUSED = 0, 1
TP_FLAG_F32_RESIDUAL = 1

# every symbol the header declares
EXPORTS = (
    "tp_mlp_w1_packed_bytes", "tp_mlp_w2_packed_bytes", "tp_mlp_pack", "tp_mlp_saved_bytes",
    "tp_mlp_fwd_workspace", "tp_mlp_fwd", "tp_mlp_bwd_workspace", "tp_mlp_bwd",
    "tp_mlp_unpack_grads", "tp_attn_wqkv_packed_bytes", "tp_attn_wo_packed_bytes",
    "tp_attn_pack", "tp_attn_fwd_workspace", "tp_attn_fwd", "tp_reduce_partials", "tp_rmsnorm",
    "tp_reduction_count", "tp_reset_reduction_count", "tp_launch_count", "tp_last_error",
    "tp_status_string", "tp_check_device_error", "tp_tensor_core_path_available", "tp_version",
    "tp_profile_enable", "tp_profile_read", "tp_profile_reset", "tp_mlp_fwd_static_ws",
    "tp_profile_read_launch",
    "tp_selftest_wait_timeout", "tp_attn_bwd_workspace", "tp_attn_bwd", "tp_attn_unpack_grads",
    "tp_reduce_scatter_partials", "tp_all_gather_slices", "tp_mlp_fwd_sp_workspace",
    "tp_mlp_fwd_sp", "tp_mlp_bwd_sp_workspace", "tp_mlp_bwd_sp", "tp_attn_fwd_sp_workspace",
    "tp_attn_fwd_sp", "tp_moe_expert_w1_bytes", "tp_moe_expert_w2_bytes",
    "tp_moe_shared_w1_bytes", "tp_moe_shared_w2_bytes", "tp_moe_pack", "tp_moe_fwd_workspace",
    "tp_moe_fwd", "tp_moe_bwd_workspace", "tp_moe_bwd", "tp_mlp_shard_sizes",
    "tp_mlp_pack_shard", "tp_mlp_fwd_shard",
    "tp_mlp_bwd_shard", "tp_attn_shard_sizes", "tp_attn_pack_shard", "tp_attn_fwd_shard",
    "tp_attn_bwd_shard", "tp_attn_bwd_sp_workspace", "tp_attn_bwd_sp",
)


class TpError(RuntimeError):
    def __init__(self, status, msg):
        super().__init__(f"{_status_name(status)}: {msg}")
        self.status = status


class tp_mlp_desc(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("d", ctypes.c_int64), ("d_ff", ctypes.c_int64),
                ("p", ctypes.c_int32), ("act", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("reduce_mode", ctypes.c_int32), ("flags", ctypes.c_int32),
                ("norm_eps", ctypes.c_float)]


class tp_moe_desc(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("d", ctypes.c_int64), ("d_ff", ctypes.c_int64),
                ("d_ff_shared", ctypes.c_int64), ("n_experts", ctypes.c_int32),
                ("top_k", ctypes.c_int32), ("p", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("flags", ctypes.c_int32), ("reserved", ctypes.c_int32)]


class tp_attn_desc(ctypes.Structure):
    _fields_ = [("b", ctypes.c_int64), ("s", ctypes.c_int64), ("h", ctypes.c_int64),
                ("n_q", ctypes.c_int32), ("n_kv", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("p", ctypes.c_int32), ("causal", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("kv_len", ctypes.c_int64), ("kv_cap", ctypes.c_int64),
                ("reduce_mode", ctypes.c_int32), ("flags", ctypes.c_int32),
                ("norm_eps", ctypes.c_float), ("reserved", ctypes.c_int32)]


class tp_shard_sizes(ctypes.Structure):
    _fields_ = [("col_weight_bytes", ctypes.c_size_t), ("row_weight_bytes", ctypes.c_size_t),
                ("saved_bytes", ctypes.c_size_t), ("fwd_workspace", ctypes.c_size_t),
                ("bwd_workspace", ctypes.c_size_t), ("partial_bytes", ctypes.c_size_t)]


_lib = None


def load():
    """Load libtpblock.so (fails loudly if it was not built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m tensor_transformer_matmul_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, S, I32, I64, F32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32, ctypes.c_int64, ctypes.c_float
    MD, AD = ctypes.POINTER(tp_mlp_desc), ctypes.POINTER(tp_attn_desc)
    ED = ctypes.POINTER(tp_moe_desc)
    sig = {
        "tp_mlp_w1_packed_bytes": (S, [MD]), "tp_mlp_w2_packed_bytes": (S, [MD]),
        "tp_mlp_pack": (I32, [MD, P, P, P, P, P, P]), "tp_mlp_saved_bytes": (S, [MD]),
        "tp_mlp_fwd_workspace": (S, [MD]),
        "tp_mlp_fwd": (I32, [MD, P, P, P, P, P, P, P, P, S, P]),
        "tp_mlp_bwd_workspace": (S, [MD]),
        "tp_mlp_bwd": (I32, [MD, P, P, P, P, P, P, P, P, P, S, P]),
        "tp_mlp_unpack_grads": (I32, [MD, P, P, P, P, P, P]),
        "tp_mlp_fwd_static_ws": (I32, [MD, P, P, P, P, P, P]),
        "tp_attn_wqkv_packed_bytes": (S, [AD]), "tp_attn_wo_packed_bytes": (S, [AD]),
        "tp_attn_pack": (I32, [AD, P, P, P, P, P, P, P]), "tp_attn_fwd_workspace": (S, [AD]),
        "tp_attn_fwd": (I32, [AD, P, P, P, P, P, P, P, P, P, S, P]),
        "tp_reduce_partials": (I32, [P, I32, I64, I32, P, P, I32, P]),
        "tp_rmsnorm": (I32, [P, I32, I64, I64, F32, P, I32, P]),
        "tp_reduction_count": (ctypes.c_uint64, []), "tp_reset_reduction_count": (None, []),
        "tp_launch_count": (ctypes.c_uint64, []), "tp_last_error": (ctypes.c_char_p, []),
        "tp_status_string": (ctypes.c_char_p, [I32]), "tp_check_device_error": (I32, [P]),
        "tp_tensor_core_path_available": (I32, []), "tp_version": (I32, []),
        "tp_selftest_wait_timeout": (I32, [ctypes.c_uint32, P]),
        "tp_attn_bwd_workspace": (S, [AD]),
        "tp_attn_bwd": (I32, [AD, P, P, P, P, P, P, P, P, S, P]),
        "tp_attn_unpack_grads": (I32, [AD, P, P, P, P, P, P, P]),
        "tp_reduce_scatter_partials": (I32, [P, I32, I64, I64, P, P, I32, P, I32, F32, P]),
        "tp_all_gather_slices": (I32, [P, I32, I64, I64, I32, P, P]),
        "tp_mlp_fwd_sp_workspace": (S, [MD]),
        "tp_mlp_fwd_sp": (I32, [MD, P, P, P, P, P, P, P, P, S, P]),
        "tp_mlp_bwd_sp_workspace": (S, [MD]),
        "tp_mlp_bwd_sp": (I32, [MD, P, P, P, P, P, P, P, P, P, S, P]),
        "tp_attn_fwd_sp_workspace": (S, [AD]),
        "tp_attn_fwd_sp": (I32, [AD, P, P, P, P, P, P, P, P, P, S, P]),
        "tp_moe_expert_w1_bytes": (S, [ED]), "tp_moe_expert_w2_bytes": (S, [ED]),
        "tp_moe_shared_w1_bytes": (S, [ED]), "tp_moe_shared_w2_bytes": (S, [ED]),
        "tp_moe_pack": (I32, [ED, P, P, P, P, P, P, P, P, P, P, P]),
        "tp_moe_fwd_workspace": (S, [ED]),
        "tp_moe_fwd": (I32, [ED, P, P, P, P, P, P, P, P, P, P, P, P, S, P]),
        "tp_moe_bwd_workspace": (S, [ED]),
        "tp_moe_bwd": (I32, [ED, P, P, P, P, P, P, P, P, P, P, P, P, P, P, S, P]),
        "tp_profile_enable": (None, [I32]), "tp_profile_reset": (None, []),
        "tp_mlp_shard_sizes": (I32, [MD, I32, ctypes.POINTER(tp_shard_sizes)]),
        "tp_mlp_pack_shard": (I32, [MD, I32, P, P, P, P, P, P]),
        "tp_mlp_fwd_shard": (I32, [MD, I32, I32, P, P, P, P, P, P, S, P]),
        "tp_mlp_bwd_shard": (I32, [MD, I32, I32, P, P, P, P, P, P, P, P, P, S, P]),
        "tp_attn_shard_sizes": (I32, [AD, I32, ctypes.POINTER(tp_shard_sizes)]),
        "tp_attn_pack_shard": (I32, [AD, I32, P, P, P, P, P, P, P]),
        "tp_attn_fwd_shard": (I32, [AD, I32, I32, P, P, P, P, P, P, P, S, P]),
        "tp_attn_bwd_shard": (I32, [AD, I32, P, P, P, P, P, P, P, P, S, P]),
        "tp_attn_bwd_sp_workspace": (S, [AD]),
        "tp_attn_bwd_sp": (I32, [AD, P, P, P, P, P, P, P, P, S, P]),
        "tp_profile_read": (I32, [I32, ctypes.c_char_p, I32, ctypes.POINTER(ctypes.c_uint64),
                                  ctypes.POINTER(ctypes.c_double)]),
        "tp_profile_read_launch": (I32, [I32, ctypes.c_int64, ctypes.POINTER(ctypes.c_double)]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _status_name(st):
    try:
        return load().tp_status_string(st).decode()
    except Exception:  # pragma: no cover
        return f"status {st}"


def _check(st):
    if st != TP_OK:
        raise TpError(st, load().tp_last_error().decode())


def _ptr(t):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch.Tensor")
    if t.numel() > 0 and not t.is_cuda:
        raise ValueError("tensor must live on the GPU")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return t.data_ptr() if t.numel() > 0 else None


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _nbytes(t):
    return 0 if t is None else t.numel() * t.element_size()


# ------------------------------------------------------------------------------------ MLP
def mlp_desc(T, d, d_ff, p, act="swiglu", dtype="bf16", reduce_mode=TP_REDUCE_SEPARATE, flags=0):
    return tp_mlp_desc(int(T), int(d), int(d_ff), int(p), ACT[act] if isinstance(act, str) else int(act),
                       DTYPE[dtype] if isinstance(dtype, str) else int(dtype), int(reduce_mode),
                       int(flags), 0.0)


def tp_mlp_w1_packed_bytes(desc):
    return load().tp_mlp_w1_packed_bytes(ctypes.byref(desc))


def tp_mlp_w2_packed_bytes(desc):
    return load().tp_mlp_w2_packed_bytes(ctypes.byref(desc))


def tp_mlp_saved_bytes(desc):
    return load().tp_mlp_saved_bytes(ctypes.byref(desc))


def tp_mlp_fwd_workspace(desc):
    return load().tp_mlp_fwd_workspace(ctypes.byref(desc))


def tp_mlp_bwd_workspace(desc):
    return load().tp_mlp_bwd_workspace(ctypes.byref(desc))


def tp_mlp_pack(desc, w1, w_up, w2, w1p, w2p, stream=None):
    _check(load().tp_mlp_pack(ctypes.byref(desc), _ptr(w1), _ptr(w_up), _ptr(w2), _ptr(w1p),
                              _ptr(w2p), _stream(stream)))


def tp_mlp_fwd(desc, x, w1p, w2p, y, residual=None, saved=None, workspace=None, stream=None,
               y_norm=None):
    _check(load().tp_mlp_fwd(ctypes.byref(desc), _ptr(x), _ptr(w1p), _ptr(w2p), _ptr(residual),
                             _ptr(y), _ptr(y_norm), _ptr(saved), _ptr(workspace),
                             _nbytes(workspace), _stream(stream)))


def tp_mlp_bwd(desc, dy, x, saved, w1p, w2p, dx, dw1p, dw2p, workspace=None, stream=None):
    _check(load().tp_mlp_bwd(ctypes.byref(desc), _ptr(dy), _ptr(x), _ptr(saved), _ptr(w1p),
                             _ptr(w2p), _ptr(dx), _ptr(dw1p), _ptr(dw2p), _ptr(workspace),
                             _nbytes(workspace), _stream(stream)))


def tp_mlp_fwd_static_ws(desc, x, w1p, w2p, y, residual=None, stream=None):
    """tp_mlp_fwd without a workspace argument, for callers that cannot allocate device memory:
    the scratch is the library's fixed 32 MiB device array (see include/tp_block.h)."""
    _check(load().tp_mlp_fwd_static_ws(ctypes.byref(desc), _ptr(x), _ptr(w1p), _ptr(w2p),
                                       _ptr(residual), _ptr(y), _stream(stream)))


def tp_mlp_unpack_grads(desc, dw1p, dw2p, dw1, dw_up, dw2, stream=None):
    _check(load().tp_mlp_unpack_grads(ctypes.byref(desc), _ptr(dw1p), _ptr(dw2p), _ptr(dw1),
                                      _ptr(dw_up), _ptr(dw2), _stream(stream)))


# ------------------------------------------------------------------------------ attention
def attn_desc(b, s, h, n_q, n_kv, head_dim, p, causal=True, dtype="bf16", kv_len=0, kv_cap=0,
              reduce_mode=TP_REDUCE_SEPARATE, flags=0):
    return tp_attn_desc(int(b), int(s), int(h), int(n_q), int(n_kv), int(head_dim), int(p),
                        int(bool(causal)), DTYPE[dtype] if isinstance(dtype, str) else int(dtype),
                        int(kv_len), int(kv_cap), int(reduce_mode), int(flags), 0.0, 0)


def tp_attn_wqkv_packed_bytes(desc):
    return load().tp_attn_wqkv_packed_bytes(ctypes.byref(desc))


def tp_attn_wo_packed_bytes(desc):
    return load().tp_attn_wo_packed_bytes(ctypes.byref(desc))


def tp_attn_fwd_workspace(desc):
    return load().tp_attn_fwd_workspace(ctypes.byref(desc))


def tp_attn_pack(desc, wq, wk, wv, wo, wqkv_p, wo_p, stream=None):
    _check(load().tp_attn_pack(ctypes.byref(desc), _ptr(wq), _ptr(wk), _ptr(wv), _ptr(wo),
                               _ptr(wqkv_p), _ptr(wo_p), _stream(stream)))


def tp_attn_fwd(desc, x, wqkv_p, wo_p, y, k_cache=None, v_cache=None, residual=None,
                workspace=None, stream=None, y_norm=None):
    _check(load().tp_attn_fwd(ctypes.byref(desc), _ptr(x), _ptr(wqkv_p), _ptr(wo_p),
                              _ptr(k_cache), _ptr(v_cache), _ptr(residual), _ptr(y),
                              _ptr(y_norm), _ptr(workspace), _nbytes(workspace),
                              _stream(stream)))


def tp_attn_bwd_workspace(desc):
    return load().tp_attn_bwd_workspace(ctypes.byref(desc))


def tp_attn_bwd(desc, x, wqkv_p, wo_p, dy, dx, dwqkv_p, dwo_p, workspace=None, stream=None):
    _check(load().tp_attn_bwd(ctypes.byref(desc), _ptr(x), _ptr(wqkv_p), _ptr(wo_p), _ptr(dy),
                              _ptr(dx), _ptr(dwqkv_p), _ptr(dwo_p), _ptr(workspace),
                              _nbytes(workspace), _stream(stream)))


def tp_attn_unpack_grads(desc, dwqkv_p, dwo_p, dwq, dwk, dwv, dwo, stream=None):
    _check(load().tp_attn_unpack_grads(ctypes.byref(desc), _ptr(dwqkv_p), _ptr(dwo_p), _ptr(dwq),
                                       _ptr(dwk), _ptr(dwv), _ptr(dwo), _stream(stream)))


# ------------------------------------------------------------------------- reduce and glue
def tp_reduce_partials(partials, p, n, out, residual=None, stream=None):
    in_t = TP_BF16 if partials.dtype == torch.bfloat16 else TP_F32
    out_t = TP_BF16 if out.dtype == torch.bfloat16 else TP_F32
    _check(load().tp_reduce_partials(_ptr(partials), int(p), int(n), in_t, _ptr(residual),
                                     _ptr(out), out_t, _stream(stream)))


def tp_rmsnorm(x, out, eps=1e-5, stream=None):
    xt = TP_BF16 if x.dtype == torch.bfloat16 else TP_F32
    ot = TP_BF16 if out.dtype == torch.bfloat16 else TP_F32
    rows = x.numel() // x.shape[-1] if x.numel() else 0
    _check(load().tp_rmsnorm(_ptr(x), xt, int(rows), int(x.shape[-1]), float(eps), _ptr(out), ot,
                             _stream(stream)))


# ------------------------------------------------------------------ one shard per device
def _pdt(partial_dtype):
    if isinstance(partial_dtype, str):
        return DTYPE[partial_dtype]
    if partial_dtype in (torch.float32, torch.bfloat16):
        return TP_BF16 if partial_dtype == torch.bfloat16 else TP_F32
    return int(partial_dtype)


def tp_mlp_shard_sizes(desc, partial_dtype="f32"):
    out = tp_shard_sizes()
    _check(load().tp_mlp_shard_sizes(ctypes.byref(desc), _pdt(partial_dtype), ctypes.byref(out)))
    return out


def tp_mlp_pack_shard(desc, shard, w1, w_up, w2, w1p_shard, w2p_shard, stream=None):
    _check(load().tp_mlp_pack_shard(ctypes.byref(desc), int(shard), _ptr(w1), _ptr(w_up),
                                    _ptr(w2), _ptr(w1p_shard), _ptr(w2p_shard), _stream(stream)))


def tp_mlp_fwd_shard(desc, shard, x, w1p_shard, w2p_shard, partial, saved=None, workspace=None,
                     stream=None):
    """partial ([T][d], its dtype is the partial dtype) = act(x W1_shard) W2_shard."""
    _check(load().tp_mlp_fwd_shard(ctypes.byref(desc), int(shard), _dt(partial), _ptr(x),
                                   _ptr(w1p_shard), _ptr(w2p_shard), _ptr(partial), _ptr(saved),
                                   _ptr(workspace), _nbytes(workspace), _stream(stream)))


def tp_mlp_bwd_shard(desc, shard, dy, x, saved, w1p_shard, w2p_shard, dx_partial, dw1p_shard,
                     dw2p_shard, workspace=None, stream=None):
    _check(load().tp_mlp_bwd_shard(ctypes.byref(desc), int(shard), _dt(dx_partial), _ptr(dy),
                                   _ptr(x), _ptr(saved), _ptr(w1p_shard), _ptr(w2p_shard),
                                   _ptr(dx_partial), _ptr(dw1p_shard), _ptr(dw2p_shard),
                                   _ptr(workspace), _nbytes(workspace), _stream(stream)))


def tp_attn_shard_sizes(desc, partial_dtype="f32"):
    out = tp_shard_sizes()
    _check(load().tp_attn_shard_sizes(ctypes.byref(desc), _pdt(partial_dtype), ctypes.byref(out)))
    return out


def tp_attn_pack_shard(desc, shard, wq, wk, wv, wo, wqkv_shard, wo_shard, stream=None):
    _check(load().tp_attn_pack_shard(ctypes.byref(desc), int(shard), _ptr(wq), _ptr(wk), _ptr(wv),
                                     _ptr(wo), _ptr(wqkv_shard), _ptr(wo_shard), _stream(stream)))


def tp_attn_fwd_shard(desc, shard, x, wqkv_shard, wo_shard, partial, k_cache=None, v_cache=None,
                      workspace=None, stream=None):
    _check(load().tp_attn_fwd_shard(ctypes.byref(desc), int(shard), _dt(partial), _ptr(x),
                                    _ptr(wqkv_shard), _ptr(wo_shard), _ptr(k_cache), _ptr(v_cache),
                                    _ptr(partial), _ptr(workspace), _nbytes(workspace),
                                    _stream(stream)))


def tp_attn_bwd_shard(desc, shard, x, wqkv_shard, wo_shard, dy, dx_partial, dwqkv_shard,
                      dwo_shard, workspace=None, stream=None):
    _check(load().tp_attn_bwd_shard(ctypes.byref(desc), int(shard), _ptr(x), _ptr(wqkv_shard),
                                    _ptr(wo_shard), _ptr(dy), _ptr(dx_partial), _ptr(dwqkv_shard),
                                    _ptr(dwo_shard), _ptr(workspace), _nbytes(workspace),
                                    _stream(stream)))


# ------------------------------------------------------------------- sequence parallelism
class _Slices:
    """A host array of device pointers, one per shard's token slice (kept alive with the
    tensors it points into)."""

    def __init__(self, tensors):
        self.tensors = list(tensors)
        self.arr = (ctypes.c_void_p * len(self.tensors))(*[_ptr(t) for t in self.tensors])

    @property
    def ptr(self):
        return ctypes.cast(self.arr, ctypes.c_void_p)


def _slices(ts):
    return None if ts is None else _Slices(ts)


def _sp(s):
    return None if s is None else s.ptr


def _dt(t):
    return TP_BF16 if t.dtype == torch.bfloat16 else TP_F32


def tp_reduce_scatter_partials(partials, p, slices, residual=None, norm=None, eps=1e-5,
                               stream=None):
    """partials [p][T][d] fp32 -> slices[i] [T/p][d] (+ residual[i]; norm[i] = RMSNorm)."""
    T, d = partials.shape[-2], partials.shape[-1]
    so, sr, sn = _Slices(slices), _slices(residual), _slices(norm)
    _check(load().tp_reduce_scatter_partials(
        _ptr(partials), int(p), int(T), int(d), _sp(sr), so.ptr, _dt(slices[0]), _sp(sn),
        _dt(norm[0]) if norm is not None else TP_F32, float(eps), _stream(stream)))


def tp_all_gather_slices(slices, out, stream=None):
    """slices[i] [R][d] -> out [p*R][d]."""
    si = _Slices(slices)
    R = slices[0].shape[0] if slices[0].dim() > 1 else 0
    d = slices[0].shape[-1]
    _check(load().tp_all_gather_slices(si.ptr, len(slices), int(R), int(d), _dt(out), _ptr(out),
                                       _stream(stream)))


def tp_mlp_fwd_sp_workspace(desc):
    return load().tp_mlp_fwd_sp_workspace(ctypes.byref(desc))


def tp_mlp_fwd_sp(desc, x_slices, w1p, w2p, y_slices, residual_slices=None, y_norm_slices=None,
                  saved=None, workspace=None, stream=None):
    xs, ys = _Slices(x_slices), _Slices(y_slices)
    rs, ns = _slices(residual_slices), _slices(y_norm_slices)
    _check(load().tp_mlp_fwd_sp(ctypes.byref(desc), xs.ptr, _ptr(w1p), _ptr(w2p), _sp(rs), ys.ptr,
                                _sp(ns), _ptr(saved), _ptr(workspace), _nbytes(workspace),
                                _stream(stream)))


def tp_mlp_bwd_sp_workspace(desc):
    return load().tp_mlp_bwd_sp_workspace(ctypes.byref(desc))


def tp_mlp_bwd_sp(desc, dy_slices, x_slices, saved, w1p, w2p, dx_slices, dw1p, dw2p,
                  workspace=None, stream=None):
    dys, xs, dxs = _Slices(dy_slices), _Slices(x_slices), _Slices(dx_slices)
    _check(load().tp_mlp_bwd_sp(ctypes.byref(desc), dys.ptr, xs.ptr, _ptr(saved), _ptr(w1p),
                                _ptr(w2p), dxs.ptr, _ptr(dw1p), _ptr(dw2p), _ptr(workspace),
                                _nbytes(workspace), _stream(stream)))


def tp_attn_fwd_sp_workspace(desc):
    return load().tp_attn_fwd_sp_workspace(ctypes.byref(desc))


def tp_attn_fwd_sp(desc, x_slices, wqkv_p, wo_p, y_slices, k_cache=None, v_cache=None,
                   residual_slices=None, y_norm_slices=None, workspace=None, stream=None):
    xs, ys = _Slices(x_slices), _Slices(y_slices)
    rs, ns = _slices(residual_slices), _slices(y_norm_slices)
    _check(load().tp_attn_fwd_sp(ctypes.byref(desc), xs.ptr, _ptr(wqkv_p), _ptr(wo_p),
                                 _ptr(k_cache), _ptr(v_cache), _sp(rs), ys.ptr, _sp(ns),
                                 _ptr(workspace), _nbytes(workspace), _stream(stream)))


def tp_attn_bwd_sp_workspace(desc):
    return load().tp_attn_bwd_sp_workspace(ctypes.byref(desc))


def tp_attn_bwd_sp(desc, x_slices, wqkv_p, wo_p, dy_slices, dx_slices, dwqkv_p, dwo_p,
                   workspace=None, stream=None):
    xs, dys, dxs = _Slices(x_slices), _Slices(dy_slices), _Slices(dx_slices)
    _check(load().tp_attn_bwd_sp(ctypes.byref(desc), xs.ptr, _ptr(wqkv_p), _ptr(wo_p), dys.ptr,
                                 dxs.ptr, _ptr(dwqkv_p), _ptr(dwo_p), _ptr(workspace),
                                 _nbytes(workspace), _stream(stream)))


# ------------------------------------------------------------------------ mixture of experts
def moe_desc(T, d, d_ff, d_ff_shared, n_experts, top_k, p):
    return tp_moe_desc(int(T), int(d), int(d_ff), int(d_ff_shared), int(n_experts), int(top_k),
                       int(p), TP_BF16, 0, 0)


def tp_moe_expert_w1_bytes(desc):
    return load().tp_moe_expert_w1_bytes(ctypes.byref(desc))


def tp_moe_expert_w2_bytes(desc):
    return load().tp_moe_expert_w2_bytes(ctypes.byref(desc))


def tp_moe_shared_w1_bytes(desc):
    return load().tp_moe_shared_w1_bytes(ctypes.byref(desc))


def tp_moe_shared_w2_bytes(desc):
    return load().tp_moe_shared_w2_bytes(ctypes.byref(desc))


def tp_moe_fwd_workspace(desc):
    return load().tp_moe_fwd_workspace(ctypes.byref(desc))


def tp_moe_pack(desc, wg, wu, w2, w1p, w2p, shared=None, w1p_s=None, w2p_s=None, stream=None):
    """wg, wu, w2: lists of the E experts' weights; shared: (wg_s, wu_s, w2_s) or None."""
    g, u, o = _Slices(wg), _Slices(wu), _Slices(w2)
    sg, su, so = shared if shared is not None else (None, None, None)
    _check(load().tp_moe_pack(ctypes.byref(desc), g.ptr, u.ptr, o.ptr, _ptr(sg), _ptr(su),
                              _ptr(so), _ptr(w1p), _ptr(w2p), _ptr(w1p_s), _ptr(w2p_s),
                              _stream(stream)))


def tp_moe_fwd(desc, x, wr, w1p, w2p, y, w1p_s=None, w2p_s=None, bias=None, residual=None,
               route_idx=None, route_w=None, workspace=None, stream=None):
    _check(load().tp_moe_fwd(ctypes.byref(desc), _ptr(x), _ptr(wr), _ptr(w1p), _ptr(w2p),
                             _ptr(w1p_s), _ptr(w2p_s), _ptr(bias), _ptr(residual), _ptr(y),
                             _ptr(route_idx), _ptr(route_w), _ptr(workspace), _nbytes(workspace),
                             _stream(stream)))


def tp_moe_bwd_workspace(desc):
    return load().tp_moe_bwd_workspace(ctypes.byref(desc))


def tp_moe_bwd(desc, x, wr, w1p, w2p, dy, dx, dwr, dw1p, dw2p, w1p_s=None, w2p_s=None,
               dw1p_s=None, dw2p_s=None, workspace=None, stream=None):
    """dwr [d][E], dw1p / dw2p (E experts' packed layouts) and dw1p_s / dw2p_s: float32."""
    _check(load().tp_moe_bwd(ctypes.byref(desc), _ptr(x), _ptr(wr), _ptr(w1p), _ptr(w2p),
                             _ptr(w1p_s), _ptr(w2p_s), _ptr(dy), _ptr(dx), _ptr(dwr), _ptr(dw1p),
                             _ptr(dw2p), _ptr(dw1p_s), _ptr(dw2p_s), _ptr(workspace),
                             _nbytes(workspace), _stream(stream)))


# ------------------------------------------------------------------------------ diagnostics
def tp_reduction_count():
    return load().tp_reduction_count()


def tp_reset_reduction_count():
    load().tp_reset_reduction_count()


def tp_launch_count():
    return load().tp_launch_count()


def tp_last_error():
    return load().tp_last_error().decode()


def tp_check_device_error(stream=None):
    _check(load().tp_check_device_error(_stream(stream)))


def tp_selftest_wait_timeout(limit_us, stream=None):
    _check(load().tp_selftest_wait_timeout(limit_us, _stream(stream)))


def tp_tensor_core_path_available():
    return bool(load().tp_tensor_core_path_available())


def tp_version():
    return load().tp_version()


def tp_profile_enable(on=True):
    load().tp_profile_enable(1 if on else 0)


def tp_profile_reset():
    load().tp_profile_reset()


def tp_profile_read():
    """{label: (launches, total_ms)} of the kernels recorded while profiling was enabled."""
    lib = load()
    out = {}
    buf = ctypes.create_string_buffer(128)
    n = ctypes.c_uint64()
    ms = ctypes.c_double()
    i = 0
    while lib.tp_profile_read(i, buf, 128, ctypes.byref(n), ctypes.byref(ms)):
        out[buf.value.decode()] = (int(n.value), float(ms.value))
        i += 1
    return out


def tp_profile_launch_ms(label):
    """Per-launch durations (ms, in launch order) of the kernel ``label`` recorded while profiling
    was enabled; [] if it was not launched."""
    lib = load()
    names = list(tp_profile_read())
    if label not in names:
        return []
    i = names.index(label)
    out = []
    ms = ctypes.c_double()
    while lib.tp_profile_read_launch(i, len(out), ctypes.byref(ms)):
        out.append(float(ms.value))
    return out
