"""ctypes binding of libmole (include/mole.h): same entry-point names, argument
marshalling only.  Every step of the computation runs in the library's CUDA
kernels; PyTorch supplies device memory and the current stream.

Importing this module loads ``libmole.so`` from this package directory and
raises ``ImportError`` if it is missing -- there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmole.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"libmole.so not found at {LIB_PATH}; build it with "
        "`python -m mixture_lookup_experts_b200._build` (nvcc, sm_100a)")

lib = ctypes.CDLL(LIB_PATH)

MOLE_OK = 0
STATUS = {0: "MOLE_OK", 1: "MOLE_ERR_ARG", 2: "MOLE_ERR_ALIGN", 3: "MOLE_ERR_UNSUPPORTED",
          4: "MOLE_ERR_WORKSPACE", 5: "MOLE_ERR_INDEX", 6: "MOLE_ERR_CUDA", 7: "MOLE_ERR_TIMEOUT",
          8: "MOLE_ERR_NO_DEVICE"}
F32, BF16 = 0, 1
ACT = {"gelu": 0, "gelu_erf": 0, "gelu_tanh": 1, "relu": 2, "silu": 3, "identity": 4}

# Every function include/mole.h declares, with its ctypes signature.
_P, _I64, _I32, _I, _SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_int, ctypes.c_size_t
SIGNATURES = {
    "mole_status_str": ([_I], ctypes.c_char_p),
    "mole_version": ([], _I),
    "mole_build_lut_workspace": ([_I64, _I64, _I32, _I64, _I, _I32], _SZ),
    "mole_build_lut": ([_P, _P, _P, _I64, _I64, _I32, _I64, _I, _I, _P, _P, _SZ, _P], _I),
    "mole_build_lut_noalloc": ([_P, _P, _P, _I64, _I64, _I32, _I64, _I, _I, _P, _P], _I),
    "mole_lookup_combine": ([_P, _I64, _P, _P, _P, _I64, _I32, _I64, _I, _P, _P], _I),
    "mole_token_groups_workspace": ([_I64, _I32], _SZ),
    "mole_token_groups_build": ([_P, _I64, _I64, _I32, _P, _SZ, _P], _I),
    "mole_lookup_combine_groups": ([_P, _I64, _P, _SZ, _P, _P, _P, _I64, _I32, _I64, _I, _P, _P], _I),
    "mole_lookup_combine_grouped_workspace": ([_I64, _I32], _SZ),
    "mole_lookup_combine_grouped": ([_P, _I64, _P, _P, _P, _I64, _I32, _I64, _I, _P, _P, _SZ, _P], _I),
    "mole_quantize_lut_nf3": ([_P, _I64, _I32, _I64, _P, _P, _P], _I),
    "mole_lookup_combine_nf3": ([_P, _I64, _P, _P, _P, _P, _I64, _I32, _I64, _I, _P, _P], _I),
    "mole_lookup_combine_nf3_groups": ([_P, _I64, _P, _SZ, _P, _P, _P, _P, _I64, _I32, _I64, _I, _P, _P], _I),
    "mole_offload_staging_bytes": ([_I64, _I64, _I32, _I64, _I, _I32], _SZ),
    "mole_offload_stage": ([_I64, _P, _SZ, _P, _P, _I64, _I32, _I64, _I, _I32, _P, _SZ, _P, _P], _I),
    "mole_lookup_combine_offload": ([_I64, _P, _SZ, _P, _P, _P, _SZ, _I64, _I32, _I64, _I, _I32, _P, _P], _I),
    "mole_shared_ffn_workspace": ([_I64, _I64], _SZ),
    "mole_shared_ffn": ([_P, _P, _P, _I64, _I64, _I64, _I, _P, _P, _P, _P, _SZ, _P], _I),
    "mole_ffn_block_workspace": ([_I64, _I64, _I64], _SZ),
    "mole_ffn_block": ([_P, _I64, _P, _SZ, _P, _P, _P, _I64, _I32, _P, _P, _I64, _I64, _I, _P, _P, _P, _SZ, _P], _I),
    "mole_build_lut_nf3": ([_P, _P, _P, _I64, _I64, _I32, _I64, _I, _P, _P, _P, _SZ, _P], _I),
    "mole_train_cache_bytes": ([_I64, _I64, _I32, _I64, _I64], _SZ),
    "mole_train_forward": ([_P, _I64, _P, _SZ, _P, _P, _P, _P, _P, _I64, _I32, _I64, _I64, _I, _P, _P, _SZ, _P, _P],
                           _I),
    "mole_train_backward": ([_P, _I64, _P, _SZ, _P, _P, _P, _P, _P, _I64, _I32, _I64, _I64, _I, _P, _P, _SZ, _I32,
                             _P, _P, _P, _P, _P, _P], _I),
    "mole_nf3_levels": ([_P], None),
    "mole_nf3_midpoints": ([_P], None),
    "mole_gather_plan": ([_P, _I64, _I64, _P, _P, _P, _P], _I),
    "mole_prefetch_rows": ([_P, _I64, _P, _I32, _I64, _I64, _P], _I),
    "mole_check": ([_P, _I], _I),
}
for _name, (_args, _res) in SIGNATURES.items():
    _fn = getattr(lib, _name)
    _fn.argtypes = _args
    _fn.restype = _res


class MoleError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)} "
                         f"({lib.mole_status_str(status).decode()})")


def _ok(status: int, where: str) -> None:
    if status != MOLE_OK:
        raise MoleError(status, where)


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _ptr(t):
    return None if t is None else t.data_ptr()


def _contig(*ts):
    for t in ts:
        if t is not None and not t.is_contiguous():
            raise ValueError("tensors must be contiguous")


def mole_version() -> int:
    return lib.mole_version()


def mole_status_str(status: int) -> str:
    return lib.mole_status_str(status).decode()


def mole_build_lut_workspace(V: int, D: int, N: int, Dr: int, dtype=torch.bfloat16,
                             experts_per_launch: int = 0) -> int:
    dt = BF16 if dtype == torch.bfloat16 else F32
    return int(lib.mole_build_lut_workspace(V, D, N, Dr, dt, experts_per_launch))


def mole_build_lut(embed: torch.Tensor, W1: torch.Tensor, W2: torch.Tensor, act: str = "gelu",
                   lut: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                   stream=None) -> torch.Tensor:
    """LUT[v, j, :] = act(E[v] . W1[j]) . W2[j] on the device (see mole.h)."""
    _contig(embed, W1, W2, lut, workspace)
    V, D = embed.shape
    N, D2, Dr = W1.shape
    if D2 != D or tuple(W2.shape) != (N, Dr, D):
        raise ValueError("shape mismatch: embed [V,D], W1 [N,D,Dr], W2 [N,Dr,D]")
    dt = _dt(embed)
    if lut is None:
        lut = torch.empty((V, N, D), dtype=embed.dtype, device=embed.device)
    if workspace is None:
        nbytes = mole_build_lut_workspace(V, D, N, Dr, embed.dtype, 0)
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=embed.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    _ok(lib.mole_build_lut(_ptr(embed), _ptr(W1), _ptr(W2), V, D, N, Dr, ACT[act], dt, _ptr(lut),
                           _ptr(workspace), ws_bytes, _stream(stream)), "mole_build_lut")
    return lut


def mole_build_lut_noalloc(embed: torch.Tensor, W1: torch.Tensor, W2: torch.Tensor, act: str = "gelu",
                           lut: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """mole_build_lut with the scratch in the library's fixed device array
    (no allocation inside the call; see mole.h for the size limit)."""
    _contig(embed, W1, W2, lut)
    V, D = embed.shape
    N, D2, Dr = W1.shape
    if D2 != D or tuple(W2.shape) != (N, Dr, D):
        raise ValueError("shape mismatch: embed [V,D], W1 [N,D,Dr], W2 [N,Dr,D]")
    if lut is None:
        lut = torch.empty((V, N, D), dtype=embed.dtype, device=embed.device)
    _ok(lib.mole_build_lut_noalloc(_ptr(embed), _ptr(W1), _ptr(W2), V, D, N, Dr, ACT[act], _dt(embed), _ptr(lut),
                                   _stream(stream)), "mole_build_lut_noalloc")
    return lut


def mole_lookup_combine(ids: torch.Tensor, h: torch.Tensor, Wr: torch.Tensor, lut: torch.Tensor,
                        out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """out[t] = sum_j softmax(h[t] . Wr)_j LUT[ids[t], j] (fp32 out; see mole.h)."""
    _contig(ids, h, Wr, lut, out)
    V, N, D = lut.shape
    T = ids.numel()
    if out is None:
        out = torch.empty((T, D), dtype=torch.float32, device=h.device)
    _ok(lib.mole_lookup_combine(_ptr(ids), T, _ptr(h), _ptr(Wr), _ptr(lut), V, N, D, _dt(h), _ptr(out),
                                _stream(stream)), "mole_lookup_combine")
    return out


def mole_token_groups_workspace(T: int, N: int) -> int:
    return int(lib.mole_token_groups_workspace(T, N))


def mole_token_groups_build(ids: torch.Tensor, V: int, N: int, groups: torch.Tensor | None = None,
                            stream=None) -> torch.Tensor:
    """Groups the batch's tokens by id (once per batch; serves every layer
    with N experts).  Returns the groups buffer (see mole.h)."""
    _contig(ids, groups)
    T = ids.numel()
    if groups is None:
        groups = torch.empty(max(1, mole_token_groups_workspace(T, N)), dtype=torch.uint8, device=ids.device)
    nbytes = groups.numel() * groups.element_size()
    _ok(lib.mole_token_groups_build(_ptr(ids), T, V, N, _ptr(groups), nbytes, _stream(stream)),
        "mole_token_groups_build")
    return groups


def mole_lookup_combine_groups(ids: torch.Tensor, groups: torch.Tensor, h: torch.Tensor, Wr: torch.Tensor,
                               lut: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """mole_lookup_combine over a grouping built from the same ids (each
    distinct row block read once); same result bit for bit (see mole.h)."""
    _contig(ids, groups, h, Wr, lut, out)
    V, N, D = lut.shape
    T = ids.numel()
    if out is None:
        out = torch.empty((T, D), dtype=torch.float32, device=h.device)
    nbytes = groups.numel() * groups.element_size()
    _ok(lib.mole_lookup_combine_groups(_ptr(ids), T, _ptr(groups), nbytes, _ptr(h), _ptr(Wr), _ptr(lut), V, N, D,
                                       _dt(h), _ptr(out), _stream(stream)), "mole_lookup_combine_groups")
    return out


def mole_lookup_combine_grouped_workspace(T: int, N: int) -> int:
    return int(lib.mole_lookup_combine_grouped_workspace(T, N))


def mole_lookup_combine_grouped(ids: torch.Tensor, h: torch.Tensor, Wr: torch.Tensor, lut: torch.Tensor,
                                out: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                                stream=None) -> torch.Tensor:
    """mole_lookup_combine with tokens grouped by id (each distinct row block
    fetched once per batch); same result bit for bit (see mole.h)."""
    _contig(ids, h, Wr, lut, out, workspace)
    V, N, D = lut.shape
    T = ids.numel()
    if out is None:
        out = torch.empty((T, D), dtype=torch.float32, device=h.device)
    if workspace is None:
        workspace = torch.empty(max(1, mole_lookup_combine_grouped_workspace(T, N)), dtype=torch.uint8,
                                device=h.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    _ok(lib.mole_lookup_combine_grouped(_ptr(ids), T, _ptr(h), _ptr(Wr), _ptr(lut), V, N, D, _dt(h), _ptr(out),
                                        _ptr(workspace), ws_bytes, _stream(stream)), "mole_lookup_combine_grouped")
    return out


def mole_quantize_lut_nf3(lut: torch.Tensor, codes: torch.Tensor | None = None,
                          scales: torch.Tensor | None = None, stream=None):
    """NF3 codes [V, N, D/64, 24] uint8 and fp16 scales [V, N, D/64] (see mole.h)."""
    _contig(lut, codes, scales)
    V, N, D = lut.shape
    if codes is None:
        codes = torch.empty((V, N, D // 64, 24), dtype=torch.uint8, device=lut.device)
    if scales is None:
        scales = torch.empty((V, N, D // 64), dtype=torch.float16, device=lut.device)
    _ok(lib.mole_quantize_lut_nf3(_ptr(lut), V, N, D, _ptr(codes), _ptr(scales), _stream(stream)),
        "mole_quantize_lut_nf3")
    return codes, scales


def mole_build_lut_nf3(embed: torch.Tensor, W1: torch.Tensor, W2: torch.Tensor, act: str = "gelu",
                       codes: torch.Tensor | None = None, scales: torch.Tensor | None = None,
                       workspace: torch.Tensor | None = None, stream=None):
    """The table build with the NF3 quantiser in its epilogue: codes
    [V, N, D/64, 24] uint8 and fp16 scales [V, N, D/64] (see mole.h)."""
    _contig(embed, W1, W2, codes, scales, workspace)
    V, D = embed.shape
    N, _, Dr = W1.shape
    if codes is None:
        codes = torch.empty((V, N, D // 64, 24), dtype=torch.uint8, device=embed.device)
    if scales is None:
        scales = torch.empty((V, N, D // 64), dtype=torch.float16, device=embed.device)
    if workspace is None:
        workspace = torch.empty(mole_build_lut_workspace(V, D, N, Dr, torch.bfloat16, 0), dtype=torch.uint8,
                                device=embed.device)
    _ok(lib.mole_build_lut_nf3(_ptr(embed), _ptr(W1), _ptr(W2), V, D, N, Dr, ACT[act], _ptr(codes), _ptr(scales),
                               _ptr(workspace), workspace.numel(), _stream(stream)), "mole_build_lut_nf3")
    return codes, scales


def mole_lookup_combine_nf3(ids: torch.Tensor, h: torch.Tensor, Wr: torch.Tensor, codes: torch.Tensor,
                            scales: torch.Tensor, out: torch.Tensor | None = None, stream=None):
    _contig(ids, h, Wr, codes, scales, out)
    V, N, nb, _ = codes.shape
    D = nb * 64
    T = ids.numel()
    if out is None:
        out = torch.empty((T, D), dtype=torch.float32, device=h.device)
    _ok(lib.mole_lookup_combine_nf3(_ptr(ids), T, _ptr(h), _ptr(Wr), _ptr(codes), _ptr(scales), V, N, D,
                                    _dt(h), _ptr(out), _stream(stream)), "mole_lookup_combine_nf3")
    return out


def mole_lookup_combine_nf3_groups(ids: torch.Tensor, groups: torch.Tensor, h: torch.Tensor, Wr: torch.Tensor,
                                   codes: torch.Tensor, scales: torch.Tensor, out: torch.Tensor | None = None,
                                   stream=None):
    """mole_lookup_combine_nf3 over a grouping built from the same ids (each
    distinct code block read and decoded once); same result bit for bit."""
    _contig(ids, groups, h, Wr, codes, scales, out)
    V, N, nb, _ = codes.shape
    D = nb * 64
    T = ids.numel()
    if out is None:
        out = torch.empty((T, D), dtype=torch.float32, device=h.device)
    nbytes = groups.numel() * groups.element_size()
    _ok(lib.mole_lookup_combine_nf3_groups(_ptr(ids), T, _ptr(groups), nbytes, _ptr(h), _ptr(Wr), _ptr(codes),
                                           _ptr(scales), V, N, D, _dt(h), _ptr(out), _stream(stream)),
        "mole_lookup_combine_nf3_groups")
    return out


def mole_offload_staging_bytes(T: int, V: int, N: int, D: int, dtype=torch.bfloat16, nf3: bool = False) -> int:
    dt = BF16 if dtype == torch.bfloat16 else F32
    return int(lib.mole_offload_staging_bytes(T, V, N, D, dt, int(nf3)))


def _table_shape(table: torch.Tensor, scales: torch.Tensor | None):
    """(V, N, D, nf3) of a [V, N, D] table or NF3 codes [V, N, D/64, 24]."""
    if scales is None:
        V, N, D = table.shape
        return V, N, D, False
    V, N, nb, _ = table.shape
    return V, N, nb * 64, True


def mole_offload_stage(T: int, groups: torch.Tensor, table: torch.Tensor, scales: torch.Tensor | None = None,
                       staging: torch.Tensor | None = None, n_rows: torch.Tensor | None = None,
                       device=None, stream=None) -> torch.Tensor:
    """Copies the batch's distinct row blocks of `table` (pinned host memory;
    with `scales`, NF3 codes and scales) into a device staging buffer, by
    the dense index the grouping gave each id (see mole.h)."""
    _contig(groups, table, scales, staging, n_rows)
    V, N, D, nf3 = _table_shape(table, scales)
    dtype = torch.bfloat16 if nf3 else table.dtype
    if staging is None:
        nbytes = max(1, mole_offload_staging_bytes(T, V, N, D, dtype, nf3))
        staging = torch.empty(nbytes, dtype=torch.uint8, device=device if device is not None else groups.device)
    _ok(lib.mole_offload_stage(T, _ptr(groups), groups.numel(), _ptr(table), _ptr(scales), V, N, D,
                               BF16 if dtype == torch.bfloat16 else F32, int(nf3), _ptr(staging), staging.numel(),
                               _ptr(n_rows), _stream(stream)), "mole_offload_stage")
    return staging


def mole_lookup_combine_offload(groups: torch.Tensor, h: torch.Tensor, Wr: torch.Tensor, staging: torch.Tensor,
                                V: int, nf3: bool = False, out: torch.Tensor | None = None,
                                stream=None) -> torch.Tensor:
    """mole_lookup_combine (nf3: mole_lookup_combine_nf3) over the rows that
    mole_offload_stage put into `staging`; same result bit for bit."""
    _contig(groups, h, Wr, staging, out)
    T, D = h.shape
    N = Wr.shape[1]
    if out is None:
        out = torch.empty((T, D), dtype=torch.float32, device=h.device)
    _ok(lib.mole_lookup_combine_offload(T, _ptr(groups), groups.numel(), _ptr(h), _ptr(Wr), _ptr(staging),
                                        staging.numel(), V, N, D, _dt(h), int(nf3), _ptr(out), _stream(stream)),
        "mole_lookup_combine_offload")
    return out


def mole_shared_ffn_workspace(T: int, Ds: int) -> int:
    return int(lib.mole_shared_ffn_workspace(T, Ds))


def mole_shared_ffn(h: torch.Tensor, W1s: torch.Tensor, W2s: torch.Tensor, act: str = "gelu",
                    add: torch.Tensor | None = None, residual: torch.Tensor | None = None,
                    out: torch.Tensor | None = None, workspace: torch.Tensor | None = None, stream=None):
    """out = act(h . W1s) . W2s + add + residual (fp32; see mole.h)."""
    _contig(h, W1s, W2s, add, residual, out, workspace)
    T, D = h.shape
    Ds = W1s.shape[1]
    if out is None:
        out = torch.empty((T, D), dtype=torch.float32, device=h.device)
    if workspace is None:
        workspace = torch.empty(max(1, mole_shared_ffn_workspace(T, Ds)), dtype=torch.uint8, device=h.device)
    _ok(lib.mole_shared_ffn(_ptr(h), _ptr(W1s), _ptr(W2s), T, D, Ds, ACT[act], _ptr(add), _ptr(residual), _ptr(out),
                            _ptr(workspace), workspace.numel(), _stream(stream)), "mole_shared_ffn")
    return out


def mole_ffn_block_workspace(T: int, D: int, Ds: int) -> int:
    return int(lib.mole_ffn_block_workspace(T, D, Ds))


def mole_ffn_block(ids: torch.Tensor, groups: torch.Tensor, h: torch.Tensor, Wr: torch.Tensor, lut: torch.Tensor,
                   W1s: torch.Tensor, W2s: torch.Tensor, act: str = "gelu", residual: torch.Tensor | None = None,
                   out: torch.Tensor | None = None, workspace: torch.Tensor | None = None, stream=None):
    """out = residual + act(h . W1s) . W2s + the routed-expert mixture (see mole.h)."""
    _contig(ids, groups, h, Wr, lut, W1s, W2s, residual, out, workspace)
    V, N, D = lut.shape
    T = ids.numel()
    Ds = W1s.shape[1]
    if out is None:
        out = torch.empty((T, D), dtype=torch.float32, device=h.device)
    if workspace is None:
        workspace = torch.empty(max(1, mole_ffn_block_workspace(T, D, Ds)), dtype=torch.uint8, device=h.device)
    _ok(lib.mole_ffn_block(_ptr(ids), T, _ptr(groups), groups.numel(), _ptr(h), _ptr(Wr), _ptr(lut), V, N, _ptr(W1s),
                           _ptr(W2s), D, Ds, ACT[act], _ptr(residual), _ptr(out), _ptr(workspace), workspace.numel(),
                           _stream(stream)), "mole_ffn_block")
    return out


def mole_train_cache_bytes(T: int, V: int, N: int, D: int, Dr: int) -> int:
    return int(lib.mole_train_cache_bytes(T, V, N, D, Dr))


def mole_train_forward(ids: torch.Tensor, groups: torch.Tensor, h: torch.Tensor, Wr: torch.Tensor, E: torch.Tensor,
                       W1: torch.Tensor, W2: torch.Tensor, act: str = "gelu", out: torch.Tensor | None = None,
                       cache: torch.Tensor | None = None, stream=None):
    """(out, cache, n_distinct): one MoLE layer's training forward (see mole.h)."""
    _contig(ids, groups, h, Wr, E, W1, W2, out, cache)
    V, D = E.shape
    N, _, Dr = W1.shape
    T = ids.numel()
    if out is None:
        out = torch.empty((T, D), dtype=torch.float32, device=h.device)
    if cache is None:
        cache = torch.empty(max(1, mole_train_cache_bytes(T, V, N, D, Dr)), dtype=torch.uint8, device=h.device)
    n = ctypes.c_int32(0)
    _ok(lib.mole_train_forward(_ptr(ids), T, _ptr(groups), groups.numel(), _ptr(h), _ptr(Wr), _ptr(E), _ptr(W1),
                               _ptr(W2), V, N, D, Dr, ACT[act], _ptr(out), _ptr(cache), cache.numel(),
                               ctypes.addressof(n), _stream(stream)), "mole_train_forward")
    return out, cache, int(n.value)


def mole_train_backward(ids: torch.Tensor, groups: torch.Tensor, h: torch.Tensor, Wr: torch.Tensor, E: torch.Tensor,
                        W1: torch.Tensor, W2: torch.Tensor, dout: torch.Tensor, cache: torch.Tensor, n_distinct: int,
                        act: str = "gelu", dh=None, dWr=None, dE=None, dW1=None, dW2=None, stream=None):
    """Adds this layer's gradients of sum(out * dout) into the fp32 buffers
    given (see mole.h); returns them."""
    _contig(ids, groups, h, Wr, E, W1, W2, dout, cache, dh, dWr, dE, dW1, dW2)
    V, D = E.shape
    N, _, Dr = W1.shape
    T = ids.numel()
    _ok(lib.mole_train_backward(_ptr(ids), T, _ptr(groups), groups.numel(), _ptr(h), _ptr(Wr), _ptr(E), _ptr(W1),
                                _ptr(W2), V, N, D, Dr, ACT[act], _ptr(dout), _ptr(cache), cache.numel(), n_distinct,
                                _ptr(dh), _ptr(dWr), _ptr(dE), _ptr(dW1), _ptr(dW2), _stream(stream)),
        "mole_train_backward")
    return dh, dWr, dE, dW1, dW2


def mole_nf3_levels():
    buf = (ctypes.c_uint16 * 8)()
    lib.mole_nf3_levels(ctypes.cast(buf, ctypes.c_void_p))
    return list(buf)


def mole_nf3_midpoints():
    buf = (ctypes.c_float * 7)()
    lib.mole_nf3_midpoints(ctypes.cast(buf, ctypes.c_void_p))
    return list(buf)


def mole_gather_plan(ids: torch.Tensor, V: int, stream=None):
    """(uniq[:n], slot) of a batch's ids (see mole.h).  Synchronises to read n."""
    _contig(ids)
    T = ids.numel()
    uniq = torch.empty(max(T, 1), dtype=torch.int32, device=ids.device)
    slot = torch.empty(max(T, 1), dtype=torch.int32, device=ids.device)
    n = torch.zeros(1, dtype=torch.int32, device=ids.device)
    _ok(lib.mole_gather_plan(_ptr(ids), T, V, _ptr(uniq), _ptr(n), _ptr(slot), _stream(stream)),
        "mole_gather_plan")
    k = int(n.item())
    return uniq[:k], slot[:T]


def mole_prefetch_rows(ids: torch.Tensor, tables, stream=None) -> None:
    """L2 prefetch of the rows of `tables` (device tensors of V rows each:
    bf16 [V, N, D] tables, NF3 code [V, N, D/64, 24] and scale [V, N, D/64]
    arrays) that the step's `ids` address (see mole.h)."""
    _contig(ids, *tables)
    tables = list(tables)
    if not tables:
        return
    V = tables[0].shape[0]
    row_bytes = tables[0].numel() // V * tables[0].element_size()
    for t in tables:
        if t.shape[0] != V or t.numel() // V * t.element_size() != row_bytes:
            raise ValueError("mole_prefetch_rows: tables of one call share V and the row size")
    arr = (ctypes.c_void_p * len(tables))(*[t.data_ptr() for t in tables])
    _ok(lib.mole_prefetch_rows(_ptr(ids), ids.numel(), arr, len(tables), V, row_bytes, _stream(stream)),
        "mole_prefetch_rows")


def mole_check(stream=None, timeout_ms: int = 10000) -> int:
    """Drain the stream (bounded) and return the device error status (0 = ok)."""
    return int(lib.mole_check(_stream(stream), timeout_ms))
