"""fp64 CPU oracle for the scoring path (ctypes wrapper around oracle.cpp).

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the
benchmark's CPU-baseline leg are the only callers.  The product library never
imports this package, and this package never imports the product library.

Each wrapper returns float64 numpy arrays; inputs are the exact values the
CUDA path receives (bf16 as uint16 bit patterns, fp32, or float64 for the
finite-difference pins).
"""

from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np

_HERE = Path(__file__).resolve().parent
_SRC = _HERE / "oracle.cpp"
_LIB = _HERE / "liboracle.so"

F32, BF16, F64 = 0, 1, 2

# oracle status bits (see oracle.cpp)
TARGET_OUT_OF_RANGE = 1 << 0
TARGET_NOT_IN_SUPPORT = 1 << 1
BAD_SUPPORT_ID = 1 << 2
DUP_SUPPORT_ID = 1 << 3
NONFINITE_INPUT = 1 << 4


def build(force: bool = False) -> Path:
    """Compile oracle.cpp into liboracle.so (g++, OpenMP)."""
    if force or not _LIB.exists() or _LIB.stat().st_mtime < _SRC.stat().st_mtime:
        tmp = _LIB.with_suffix(f".so.tmp{os.getpid()}")
        subprocess.run(["g++", "-O2", "-std=c++17", "-ffp-contract=off", "-fopenmp", "-shared", "-fPIC", "-o",
                        str(tmp), str(_SRC)], check=True)
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        _lib = ctypes.CDLL(str(_LIB))
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _dtype_code(a: np.ndarray) -> int:
    if a.dtype == np.uint16:
        return BF16
    if a.dtype == np.float32:
        return F32
    if a.dtype == np.float64:
        return F64
    raise TypeError(f"unsupported logits dtype {a.dtype}")


def _row_param(v, rows, dt):
    """Returns (array-or-None, scalar)."""
    if v is None:
        return None, 0
    if np.isscalar(v):
        return None, v
    a = np.ascontiguousarray(v, dtype=dt)
    assert a.shape == (rows,)
    return a, 0


def score(logits, targets, temperature=1.0, top_k=0, top_p=1.0, min_p=0.0,
          support=None, want_mask=False, vocab=None):
    """Score every row.  Returns a dict of per-row arrays (and the mask)."""
    logits = np.ascontiguousarray(logits)
    rows, ld = logits.shape
    vocab = ld if vocab is None else vocab
    targets = np.ascontiguousarray(targets, dtype=np.int32)
    t_arr, t_s = _row_param(temperature, rows, np.float64)
    k_arr, k_s = _row_param(top_k, rows, np.int32)
    p_arr, p_s = _row_param(top_p, rows, np.float64)
    m_arr, m_s = _row_param(min_p, rows, np.float64)
    width, sld = 0, 0
    if support is not None:
        support = np.ascontiguousarray(support, dtype=np.int32)
        width = sld = support.shape[1]
    out = {k: np.empty(rows, np.float64) for k in
           ("lp_full", "lp_support", "h_full", "h_support", "topp_margin", "minp_margin",
            "topk_gap", "lse_full")}
    valid = np.empty(rows, np.uint8)
    status = np.empty(rows, np.uint32)
    size = np.empty(rows, np.int32)
    mask = np.empty((rows, vocab), np.uint8) if want_mask else None
    L = lib()
    L.vso_score.restype = ctypes.c_int
    rc = L.vso_score(
        ctypes.c_int(rows), ctypes.c_int(vocab), ctypes.c_int64(ld),
        ctypes.c_int(_dtype_code(logits)), _ptr(logits), _ptr(t_arr), ctypes.c_double(t_s),
        _ptr(targets), _ptr(k_arr), ctypes.c_int32(int(k_s)), _ptr(p_arr),
        ctypes.c_double(p_s), _ptr(m_arr), ctypes.c_double(m_s), _ptr(support),
        ctypes.c_int(width), ctypes.c_int64(sld), _ptr(out["lp_full"]),
        _ptr(out["lp_support"]), _ptr(out["h_full"]), _ptr(out["h_support"]), _ptr(valid),
        _ptr(status), _ptr(size), _ptr(mask), _ptr(out["topp_margin"]),
        _ptr(out["minp_margin"]), _ptr(out["topk_gap"]), _ptr(out["lse_full"]))
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    out.update(valid=valid, status=status, support_size=size)
    if want_mask:
        out["mask"] = mask
    return out


def prefix(logits, prefix_len, temperature=1.0, top_k=0, vocab=None, want_ids=False):
    """Facts of the first n = prefix_len[i] entries of each row's total order
    (vso_prefix): top-p masses at n and n - 1 (renormalised over the top-k
    set), min-p ratios exp(z - m) of the n-th and (n+1)-th entries, the top-k
    size, and optionally the ids (a list of arrays)."""
    logits = np.ascontiguousarray(logits)
    rows, ld = logits.shape
    vocab = ld if vocab is None else vocab
    n = np.ascontiguousarray(prefix_len, dtype=np.int32)
    assert n.shape == (rows,)
    t_arr, t_s = _row_param(temperature, rows, np.float64)
    k_arr, k_s = _row_param(top_k, rows, np.int32)
    max_ids = max(1, int(n.max(initial=0))) if want_ids else 0
    ids = np.full((rows, max_ids), -1, np.int32) if want_ids else None
    out = {k: np.empty(rows, np.float64) for k in ("mass_n", "mass_prev", "ratio_n", "ratio_next")}
    nk = np.empty(rows, np.int32)
    L = lib()
    L.vso_prefix.restype = ctypes.c_int
    rc = L.vso_prefix(ctypes.c_int(rows), ctypes.c_int(vocab), ctypes.c_int64(ld),
                      ctypes.c_int(_dtype_code(logits)), _ptr(logits), _ptr(t_arr),
                      ctypes.c_double(t_s), _ptr(k_arr), ctypes.c_int32(int(k_s)), _ptr(n),
                      _ptr(ids), ctypes.c_int(max_ids), _ptr(out["mass_n"]),
                      _ptr(out["mass_prev"]), _ptr(out["ratio_n"]), _ptr(out["ratio_next"]),
                      _ptr(nk))
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    out["nk"] = nk
    if want_ids:
        out["ids"] = [ids[i, :n[i]] for i in range(rows)]
    return out


def score_grad(logits, targets, g_lp_full=None, g_lp_support=None, g_h_full=None,
               g_h_support=None, temperature=1.0, top_k=0, top_p=1.0, min_p=0.0,
               support=None, vocab=None):
    """dL/dlogits for L = sum_i g_lpV lp_V + g_lpS lp_S + g_hV H_V + g_hS H_S."""
    logits = np.ascontiguousarray(logits)
    rows, ld = logits.shape
    vocab = ld if vocab is None else vocab
    targets = np.ascontiguousarray(targets, dtype=np.int32)
    t_arr, t_s = _row_param(temperature, rows, np.float64)
    k_arr, k_s = _row_param(top_k, rows, np.int32)
    p_arr, p_s = _row_param(top_p, rows, np.float64)
    m_arr, m_s = _row_param(min_p, rows, np.float64)
    gs = [None if g is None else np.ascontiguousarray(np.broadcast_to(g, (rows,)), np.float64)
          for g in (g_lp_full, g_lp_support, g_h_full, g_h_support)]
    width, sld = 0, 0
    if support is not None:
        support = np.ascontiguousarray(support, dtype=np.int32)
        width = sld = support.shape[1]
    d = np.empty((rows, vocab), np.float64)
    L = lib()
    rc = L.vso_score_grad(
        ctypes.c_int(rows), ctypes.c_int(vocab), ctypes.c_int64(ld),
        ctypes.c_int(_dtype_code(logits)), _ptr(logits), _ptr(t_arr), ctypes.c_double(t_s),
        _ptr(targets), _ptr(k_arr), ctypes.c_int32(int(k_s)), _ptr(p_arr),
        ctypes.c_double(p_s), _ptr(m_arr), ctypes.c_double(m_s), _ptr(support),
        ctypes.c_int(width), ctypes.c_int64(sld), *[_ptr(g) for g in gs], _ptr(d))
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    return d


def l1(draft, target, weight=None, want_grad=False, tie_eps=1e-6, vocab=None, global_wsum=None):
    """Draft/target distance; global_wsum: the weight sum over all shards of a
    row-sharded batch (the loss denominator), else this call's."""
    draft = np.ascontiguousarray(draft)
    target = np.ascontiguousarray(target)
    assert draft.dtype == target.dtype and draft.shape == target.shape
    rows, ld = draft.shape
    vocab = ld if vocab is None else vocab
    w = None if weight is None else np.ascontiguousarray(weight, np.float64)
    out = {k: np.empty(rows, np.float64) for k in ("l1", "accept")}
    nd = np.empty(3, np.float64)
    ties = np.empty(rows, np.int32)
    g = np.empty((rows, vocab), np.float64) if want_grad else None
    L = lib()
    rc = L.vso_l1(ctypes.c_int(rows), ctypes.c_int(vocab), ctypes.c_int64(ld),
                  ctypes.c_int(_dtype_code(draft)), _ptr(draft), _ptr(target), _ptr(w),
                  _ptr(out["l1"]), _ptr(out["accept"]), _ptr(nd), _ptr(g),
                  ctypes.c_double(tie_eps), _ptr(ties),
                  None if global_wsum is None else ctypes.byref(ctypes.c_double(global_wsum)))
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    out.update(loss_num=nd[0], loss_den=nd[1], loss=nd[2], near_ties=ties)
    if want_grad:
        out["grad"] = g
    return out


def lmhead_logits(hidden_bits, weight_bits, rows_sel, temperature):
    """fp64 tempered logits for the selected rows: (H[rows] . W^T) / T."""
    hidden_bits = np.ascontiguousarray(hidden_bits, np.uint16)
    weight_bits = np.ascontiguousarray(weight_bits, np.uint16)
    rows_sel = np.ascontiguousarray(rows_sel, np.int32)
    vocab, hdim = weight_bits.shape
    out = np.empty((len(rows_sel), vocab), np.float64)
    L = lib()
    rc = L.vso_lmhead_logits(ctypes.c_int(len(rows_sel)), _ptr(rows_sel), ctypes.c_int(vocab),
                             ctypes.c_int(hdim), _ptr(hidden_bits),
                             ctypes.c_int64(hidden_bits.shape[1]), _ptr(weight_bits),
                             ctypes.c_int64(hdim), ctypes.c_double(temperature), _ptr(out))
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    return out


def _wide(a):
    """bf16 bit patterns (uint16) or float64 values, widened exactly to float64."""
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def lmhead_grad(hidden, weight, targets, temperature, g_lp_full=None, g_lp_support=None,
                g_h_full=None, g_h_support=None, top_k=0, top_p=1.0, min_p=0.0, support=None):
    """Gradients of L = sum_i g_lpV lp_V + g_lpS lp_S + g_hV H_V + g_hS H_S
    with respect to the LM head's inputs (xorl issue #71, section 1: the
    projection, then the scoring op, then its VJP).  With x = H W^T
    (fp64 products of the exact inputs) and z = x / T, the logit gradient
    dz comes from score_grad on z; then dx = dz / T and
        dH = dx W,   dW = dx^T H   (numpy matmul in fp64).
    hidden [rows, hidden] and weight [vocab, hidden] are bf16 bit patterns
    or float64; temperature a scalar.  Returns (dH, dW)."""
    H = _wide(hidden)
    W = _wide(weight)
    z = (H @ W.T) / float(temperature)
    dz = score_grad(z, targets, g_lp_full, g_lp_support, g_h_full, g_h_support, temperature=1.0,
                    top_k=top_k, top_p=top_p, min_p=min_p, support=support)
    dx = dz / float(temperature)
    return dx @ W, dx.T @ H


def set_threads(n: int) -> None:
    """Set the OpenMP thread count of the oracle library."""
    os.environ["OMP_NUM_THREADS"] = str(n)
    try:
        gomp = ctypes.CDLL("libgomp.so.1")
        gomp.omp_set_num_threads(ctypes.c_int(n))
    except OSError:
        pass


def max_threads() -> int:
    try:
        gomp = ctypes.CDLL("libgomp.so.1")
        return int(gomp.omp_get_max_threads())
    except OSError:
        return 1


def philox4x64_10(counter, key):
    """One Philox4x64-10 block: four 64-bit words for a 4-word counter and a
    2-word key."""
    c = np.ascontiguousarray(counter, np.uint64)
    k = np.ascontiguousarray(key, np.uint64)
    out = np.empty(4, np.uint64)
    lib().vso_philox4x64_10(_ptr(c), _ptr(k), _ptr(out))
    return out


def log_f32(x):
    """The oracle's fp32 natural logarithm (fixed operation sequence)."""
    L = lib()
    L.vso_log_f32.restype = ctypes.c_float
    L.vso_log_f32.argtypes = [ctypes.c_float]
    return np.float32(L.vso_log_f32(float(np.float32(x))))


def gumbel_f32(seed, row, j):
    """G_j of the sampling recipe for (seed, row, token j), fp32."""
    L = lib()
    L.vso_gumbel_f32.restype = ctypes.c_float
    L.vso_gumbel_f32.argtypes = [ctypes.c_uint64, ctypes.c_int, ctypes.c_int64]
    return np.float32(L.vso_gumbel_f32(int(seed), int(row), int(j)))


def gumbel_sample(logits, temperature, mask, seed, vocab=None):
    """Seeded Gumbel-max token per row over the support `mask` ([rows, vocab]
    bytes): argmax_j fl32(l_j / T) + G_j in fp32, smallest j on ties, -1 for
    an empty support.  temperature: scalar or fp32 per row."""
    logits = np.ascontiguousarray(logits)
    rows, ld = logits.shape
    vocab = ld if vocab is None else vocab
    mask = np.ascontiguousarray(mask, np.uint8)
    t_arr = None
    t_s = 1.0
    if np.ndim(temperature):
        t_arr = np.ascontiguousarray(temperature, np.float32)
    else:
        t_s = float(np.float32(temperature))
    out = np.empty(rows, np.int32)
    L = lib()
    rc = L.vso_gumbel_sample(ctypes.c_int(rows), ctypes.c_int(vocab), ctypes.c_int64(ld),
                             ctypes.c_int(_dtype_code(logits)), _ptr(logits), _ptr(t_arr),
                             ctypes.c_float(t_s), _ptr(mask), ctypes.c_uint64(int(seed)),
                             _ptr(out))
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    return out
