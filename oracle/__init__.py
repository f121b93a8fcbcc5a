"""Oracle for the MoLE lookup path: plain, slow fp64 CPU reference.

TEST INFRASTRUCTURE ONLY.  Only the test-suite, ``__graft_entry__.smoke()`` and
the CPU-baseline / reference legs of ``bench.py`` may import this package.  The
product library never does, and shares no code with it: the arithmetic lives in
``mole_oracle.c`` (plain C, fp64), this module only marshals numpy arrays.

Source page ("MoLE page"): "ICML 2025 Spotlight | 华为诺亚提出端侧大模型新架构MoLE，
内存搬运代价降低1000倍" (zejuncao.github.io), sections 训练阶段 (training stage),
推理阶段 (inference stage), 复杂度分析 (complexity), 实验结果 (results).

Arrays: fp32 tensors are ``np.float32``; bf16 tensors are ``np.uint16`` bit
patterns.  Results are ``np.float64``.

Pins (what ties each function to something other than itself) are in
``tests/test_oracle_pins.py``.  Parity unpinned: the model-quality claims of the
page (comparable quality to MoE, NF3 "basically unchanged"), which need trained
weights; they are not computed here.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mole_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libmole_oracle.so")

F32, BF16 = 0, 1
ACT = {"gelu": 0, "gelu_erf": 0, "gelu_tanh": 1, "relu": 2, "silu": 3, "identity": 4}

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (fp64, no FMA contraction, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
               "-fno-fast-math", "-std=c11", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _L():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        P, I64, I32, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_int
        lib.oracle_build_lut.argtypes = [P, P, P, I64, I64, I32, I64, I, I, I, P, I64, P, I]
        lib.oracle_build_lut.restype = I
        lib.oracle_build_lut_ex.argtypes = [P, P, P, I64, I64, I32, I64, I, I, I, P, I64, P, P, P, I]
        lib.oracle_build_lut_ex.restype = I
        lib.oracle_round_bf16_array.argtypes = [P, P, I64]
        lib.oracle_combine.argtypes = [P, I64, P, I, P, I, P, I, I64, I32, I64, P, P, I]
        lib.oracle_combine.restype = I64
        lib.oracle_gather_plan.argtypes = [P, I64, I64, P, P, P]
        lib.oracle_gather_plan.restype = I
        lib.oracle_nf3_levels.argtypes = [P]
        lib.oracle_nf3_levels_f16.argtypes = [P]
        lib.oracle_nf3_midpoints.argtypes = [P]
        lib.oracle_quantize_nf3.argtypes = [P, I64, I32, I64, P, P]
        lib.oracle_quantize_nf3.restype = I
        lib.oracle_dequantize_nf3.argtypes = [P, P, I64, I32, I64, P]
        lib.oracle_dequantize_nf3.restype = I
        lib.oracle_nf3_code.argtypes = [P, I]
        lib.oracle_nf3_code.restype = I
        lib.oracle_combine_nf3.argtypes = [P, I64, P, I, P, I, P, P, I64, I32, I64, P, I]
        lib.oracle_combine_nf3.restype = I64
        lib.oracle_act.argtypes = [I, ctypes.c_double]
        lib.oracle_act.restype = ctypes.c_double
        lib.oracle_round_bf16.argtypes = [ctypes.c_double]
        lib.oracle_round_bf16.restype = ctypes.c_double
        lib.oracle_round_f16.argtypes = [ctypes.c_double]
        lib.oracle_round_f16.restype = ctypes.c_double
        lib.oracle_max_threads.restype = I
        _lib = lib
    return _lib


def _dtype_code(a: np.ndarray) -> int:
    if a.dtype == np.float32:
        return F32
    if a.dtype == np.uint16:
        return BF16
    raise TypeError(f"oracle takes float32 or uint16 (bf16 bits), got {a.dtype}")


def _c(a: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(a)


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def max_threads() -> int:
    return int(_L().oracle_max_threads())


def act(name: str, u: float) -> float:
    """The expert activation at one point (fp64)."""
    return float(_L().oracle_act(ACT[name], float(u)))


def round_bf16(x: float) -> float:
    return float(_L().oracle_round_bf16(float(x)))


def round_f16(x: float) -> float:
    return float(_L().oracle_round_f16(float(x)))


def build_lut(E, W1, W2, act_name: str = "gelu", round_h: bool = True, rows=None,
              nthreads: int = 0, with_allowance: bool = False):
    """LUT[v, j, :] = act(E[v] . W1[j]) . W2[j] for the requested rows (fp64).

    MoLE page, 推理阶段: the embedding matrix is fed to every routed expert.
    E [V, D], W1 [N, D, Dr], W2 [N, Dr, D]; all fp32 or all bf16 bits.
    Returns [len(rows), N, D] (or [V, N, D] when rows is None); with
    with_allowance (needs round_h) also the per-element allowance for
    ambiguous bf16 roundings of the hidden activation and their count.
    """
    if with_allowance:
        return _build_lut_ex(E, W1, W2, act_name, round_h, rows, nthreads)
    E, W1, W2 = _c(E), _c(W1), _c(W2)
    dt = _dtype_code(E)
    assert _dtype_code(W1) == dt and _dtype_code(W2) == dt
    V, D = E.shape
    N, D2, Dr = W1.shape
    assert D2 == D and W2.shape == (N, Dr, D)
    if rows is None:
        rows_arr, n_rows, rows_p = None, V, None
    else:
        rows_arr = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        n_rows, rows_p = rows_arr.size, _p(rows_arr)
    out = np.empty((n_rows, N, D), dtype=np.float64)
    rc = _L().oracle_build_lut(_p(E), _p(W1), _p(W2), V, D, N, Dr, ACT[act_name], dt,
                               1 if round_h else 0, rows_p, n_rows, _p(out), nthreads)
    if rc != 0:
        raise ValueError("oracle_build_lut: bad argument")
    return out


def _build_lut_ex(E, W1, W2, act_name, round_h, rows, nthreads):
    E, W1, W2 = _c(E), _c(W1), _c(W2)
    dt = _dtype_code(E)
    V, D = E.shape
    N, _, Dr = W1.shape
    if rows is None:
        n_rows, rows_p = V, None
    else:
        rows_arr = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        n_rows, rows_p = rows_arr.size, _p(rows_arr)
    out = np.empty((n_rows, N, D), dtype=np.float64)
    allow = np.empty((n_rows, N, D), dtype=np.float64)
    n_amb = np.zeros(1, dtype=np.int64)
    rc = _L().oracle_build_lut_ex(_p(E), _p(W1), _p(W2), V, D, N, Dr, ACT[act_name], dt, 1 if round_h else 0,
                                  rows_p, n_rows, _p(out), _p(allow), _p(n_amb), nthreads)
    if rc != 0:
        raise ValueError("oracle_build_lut_ex: bad argument")
    return out, allow, int(n_amb[0])


def ffn_block(ids, h, Wr, lut, W1s, W2s, act_name: str = "gelu", residual=None, nthreads: int = 0):
    """out[t] = residual[t] + act(h[t] . W1s) . W2s + sum_j g_j LUT[ids[t], j] in fp64.

    MoLE page, 训练阶段 / 推理阶段: at inference the shared experts remain dense
    FFNs on the previous layer's output h, and only the routed experts become
    the table; the layer output adds the residual (reading: one shared expert
    of the routed experts' form).  The shared expert is build_lut's expert
    evaluated on the rows of h (the hidden activation rounded to bf16 at the
    same point), the mixture is combine().  Returns (out [T, D], allowance of
    the shared expert's ambiguous bf16 roundings [T, D], n_bad).
    """
    T, D = h.shape
    Ds = W1s.shape[1]
    shared, allow, _ = build_lut(h, W1s.reshape(1, D, Ds), W2s.reshape(1, Ds, D), act_name, True, None, nthreads,
                                 with_allowance=True)
    mix, n_bad = combine(ids, h, Wr, lut, nthreads=nthreads)
    out = shared[:, 0, :] + mix
    if residual is not None:
        out = out + np.asarray(residual, dtype=np.float64)
    return out, allow[:, 0, :], n_bad


def _bits_f64(a):
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def _act64(name, u):
    """Expert activation on fp64 arrays (the forms of mole_oracle.c)."""
    from scipy.special import erfc
    if name in ("gelu", "gelu_erf"):
        return u * 0.5 * erfc(-u / np.sqrt(2.0))
    if name == "gelu_tanh":
        return 0.5 * u * (1.0 + np.tanh(np.sqrt(2.0 / np.pi) * (u + 0.044715 * u ** 3)))
    if name == "relu":
        return np.maximum(u, 0.0)
    if name == "silu":
        return u / (1.0 + np.exp(-u))
    return u


def _act64_grad(name, u):
    """Derivative of _act64 (the chain rule written out per activation)."""
    from scipy.special import erfc
    if name in ("gelu", "gelu_erf"):
        return 0.5 * erfc(-u / np.sqrt(2.0)) + u * np.exp(-0.5 * u * u) / np.sqrt(2.0 * np.pi)
    if name == "gelu_tanh":
        c = np.sqrt(2.0 / np.pi)
        th = np.tanh(c * (u + 0.044715 * u ** 3))
        return 0.5 * (1.0 + th) + 0.5 * u * (1.0 - th * th) * c * (1.0 + 3.0 * 0.044715 * u * u)
    if name == "relu":
        return (u > 0).astype(np.float64)
    if name == "silu":
        sg = 1.0 / (1.0 + np.exp(-u))
        return sg * (1.0 + u * (1.0 - sg))
    return np.ones_like(u)


def train_step(ids, h, Wr, E, W1, W2, act_name: str = "gelu", dout=None, round_h: bool = True,
               round_ops: bool = False):
    """One MoLE layer in training, forward and backward, in fp64 (numpy).

    MoLE page, 训练阶段: the routed experts take the token's embedding row,
    all N are active, and the router on the previous layer's output h mixes
    them:  out[t] = sum_j g_j(h[t]) f_j(E[ids[t]]),  g = softmax(h Wr),
    f_j(x) = act(x W1[j]) W2[j] with the hidden activation rounded to bf16
    when round_h (the bf16 build's precision point; the backward treats the
    rounding as identity).  Returns (out, grads) where grads holds the
    gradients of L = sum(out * dout): dh, dWr, dE, dW1, dW2 (all fp64).
    Every id must lie in [0, V).

    A routed expert's output depends on the token id alone, so the experts
    are evaluated once per distinct id and the per-token terms summed by id
    (equal to the per-token definition; a pin checks that on tiny inputs).
    round_ops (with round_h) adds the bf16 precision points of a bf16 device
    step: the expert outputs held as a bf16 table row, dL/dY (summed over a
    distinct id's tokens) and dL/dpre, each the bf16 operand of a backward
    contraction, rounded to bf16 (ties to even) where the device rounds them.
    """
    ids = np.asarray(ids, dtype=np.int64)
    hf, Wrf, Ef, W1f, W2f = (_bits_f64(x) for x in (h, Wr, E, W1, W2))
    uniq, inv = np.unique(ids, return_inverse=True)
    inv = inv.ravel()
    Eu = Ef[uniq]                                      # [U, D]
    pre = np.einsum("ud,jdr->jur", Eu, W1f)            # [N, U, Dr]
    a = _act64(act_name, pre)
    if round_h:
        a = round_bf16_array(a)
    Y = np.einsum("jur,jrd->ujd", a, W2f)              # [U, N, D]
    if round_ops:
        Y = round_bf16_array(Y)
    z = hf @ Wrf
    z = z - z.max(axis=1, keepdims=True)
    g = np.exp(z)
    g /= g.sum(axis=1, keepdims=True)
    out = np.einsum("tj,tjd->td", g, Y[inv])
    grads = None
    if dout is not None:
        do = np.asarray(dout, dtype=np.float64)
        dg = np.einsum("td,tjd->tj", do, Y[inv])
        dz = g * (dg - (g * dg).sum(axis=1, keepdims=True))
        dY = np.zeros_like(Y)
        np.add.at(dY, inv, g[:, :, None] * do[:, None, :])
        if round_ops:
            dY = round_bf16_array(dY)
        dA = np.einsum("ujd,jrd->jur", dY, W2f)
        dpre = dA * _act64_grad(act_name, pre)
        if round_ops:
            dpre = round_bf16_array(dpre)
        dE = np.zeros_like(Ef)
        dE[uniq] = np.einsum("jur,jdr->ud", dpre, W1f)
        grads = {"dh": dz @ Wrf.T, "dWr": hf.T @ dz, "dE": dE,
                 "dW1": np.einsum("ud,jur->jdr", Eu, dpre), "dW2": np.einsum("jur,ujd->jrd", a, dY)}
    return out, grads


def round_bf16_array(x: np.ndarray) -> np.ndarray:
    """Element-wise bf16 rounding (ties to even) of float64 values."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    y = np.empty_like(x)
    _L().oracle_round_bf16_array(_p(x), _p(y), x.size)
    return y


def combine(ids, h, Wr, lut, V: int | None = None, nthreads: int = 0, return_gates=False):
    """out[t] = sum_j softmax(h[t] . Wr)_j LUT[ids[t], j] in fp64.

    MoLE page, 训练阶段 (router on the previous layer's output, all routed
    experts active) and 推理阶段 (rows addressed by token id).
    Returns (out [T, D] float64, n_bad) or (out, gates, n_bad).
    """
    ids = _c(np.asarray(ids, dtype=np.int32))
    h, Wr, lut = _c(h), _c(Wr), _c(lut)
    T = ids.size
    Vl, N, D = lut.shape
    V = Vl if V is None else V
    assert h.shape == (T, D) and Wr.shape == (D, N)
    out = np.empty((T, D), dtype=np.float64)
    gates = np.empty((T, N), dtype=np.float64)
    n_bad = _L().oracle_combine(_p(ids), T, _p(h), _dtype_code(h), _p(Wr), _dtype_code(Wr),
                                _p(lut), _dtype_code(lut), V, N, D, _p(out), _p(gates), nthreads)
    if n_bad < 0:
        raise ValueError("oracle_combine: bad argument")
    return (out, gates, int(n_bad)) if return_gates else (out, int(n_bad))


def gather_plan(ids, V: int):
    """Sorted distinct ids of a batch and each token's slot among them."""
    ids = _c(np.asarray(ids, dtype=np.int32))
    T = ids.size
    uniq = np.zeros(max(T, 1), dtype=np.int32)
    slot = np.zeros(max(T, 1), dtype=np.int32)
    n = np.zeros(1, dtype=np.int32)
    rc = _L().oracle_gather_plan(_p(ids), T, V, _p(uniq), _p(n), _p(slot))
    if rc != 0:
        raise ValueError("oracle_gather_plan: id out of range")
    return uniq[: int(n[0])].copy(), slot[:T].copy()


def nf3_levels() -> np.ndarray:
    """The NormalFloat k=3 levels from the construction, in fp64 (ascending)."""
    lv = np.zeros(8, dtype=np.float64)
    _L().oracle_nf3_levels(_p(lv))
    return lv


def nf3_levels_f16() -> np.ndarray:
    """The stored levels: fp16 bit patterns (uint16)."""
    b = np.zeros(8, dtype=np.uint16)
    _L().oracle_nf3_levels_f16(_p(b))
    return b


def nf3_midpoints() -> np.ndarray:
    m = np.zeros(7, dtype=np.float32)
    _L().oracle_nf3_midpoints(_p(m))
    return m


def quantize_nf3(lut_bf16: np.ndarray):
    """Codes [V, N, D/64, 24] u8 and fp16 scale bits [V, N, D/64] u16."""
    lut_bf16 = _c(lut_bf16)
    assert lut_bf16.dtype == np.uint16
    V, N, D = lut_bf16.shape
    codes = np.zeros((V, N, D // 64, 24), dtype=np.uint8)
    scales = np.zeros((V, N, D // 64), dtype=np.uint16)
    rc = _L().oracle_quantize_nf3(_p(lut_bf16), V, N, D, _p(codes), _p(scales))
    if rc != 0:
        raise ValueError("oracle_quantize_nf3: bad argument")
    return codes, scales


def nf3_code(block: np.ndarray, e: int) -> int:
    block = _c(np.asarray(block, dtype=np.uint8))
    assert block.size == 24
    return int(_L().oracle_nf3_code(_p(block), e))


def dequantize_nf3(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    codes, scales = _c(codes), _c(scales)
    V, N, nb, _ = codes.shape
    D = nb * 64
    out = np.empty((V, N, D), dtype=np.float64)
    rc = _L().oracle_dequantize_nf3(_p(codes), _p(scales), V, N, D, _p(out))
    if rc != 0:
        raise ValueError("oracle_dequantize_nf3: bad argument")
    return out


def combine_nf3(ids, h, Wr, codes, scales, nthreads: int = 0):
    """oracle_combine over an NF3 table (levels times block scales, exact)."""
    ids = _c(np.asarray(ids, dtype=np.int32))
    h, Wr, codes, scales = _c(h), _c(Wr), _c(codes), _c(scales)
    T = ids.size
    V, N, nb, _ = codes.shape
    D = nb * 64
    assert h.shape == (T, D) and Wr.shape == (D, N) and scales.shape == (V, N, nb)
    out = np.empty((T, D), dtype=np.float64)
    n_bad = _L().oracle_combine_nf3(_p(ids), T, _p(h), _dtype_code(h), _p(Wr), _dtype_code(Wr),
                                    _p(codes), _p(scales), V, N, D, _p(out), nthreads)
    if n_bad < 0:
        raise ValueError("oracle_combine_nf3: bad argument")
    return out, int(n_bad)
