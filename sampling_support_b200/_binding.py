"""ctypes binding of libvs.so: argument marshalling only.

Every step of the scoring path runs in the library's CUDA kernels; this
module builds the argument structs from torch tensors (device memory and
streams come from PyTorch), calls the C ABI, and raises on a non-zero status.
There is no fallback: if libvs.so cannot be loaded, every call raises.
"""

from __future__ import annotations

import ctypes
from pathlib import Path

import torch

_PKG = Path(__file__).resolve().parent
LIB_PATH = _PKG / "libvs.so"

VS_OK, VS_ERR_INVALID_ARG, VS_ERR_UNSUPPORTED, VS_ERR_WORKSPACE, VS_ERR_CUDA = 0, 1, 2, 3, 4
VS_F32, VS_BF16 = 0, 1
VS_WANT_ENTROPY, VS_WANT_SUPPORT_MASK, VS_WANT_GRAD, VS_WANT_SAMPLE = 1, 2, 4, 8
VS_GRAD_DENSE, VS_GRAD_ACCUMULATE, VS_GRAD_SPARSE = 0, 1, 2
VS_CTX_BYTES_PER_ROW = 64
VS_MAX_SUPPORT_WIDTH = 1024
VS_MAX_FUSED_TOPK = 64

ROW_TARGET_OUT_OF_RANGE = 1 << 0
ROW_TARGET_NOT_IN_SUPPORT = 1 << 1
ROW_BAD_SUPPORT_ID = 1 << 2
ROW_DUP_SUPPORT_ID = 1 << 3
ROW_NONFINITE_INPUT = 1 << 4
ROW_DEVICE_TIMEOUT = 1 << 5
ROW_EMPTY_SUPPORT = 1 << 6

_vp = ctypes.c_void_p


class ScoreArgs(ctypes.Structure):
    _fields_ = [
        ("rows", ctypes.c_int32), ("vocab", ctypes.c_int32), ("ld", ctypes.c_int64),
        ("dtype", ctypes.c_int32), ("logits", _vp),
        ("temperature", _vp), ("temperature_scalar", ctypes.c_float),
        ("targets", _vp),
        ("top_k", _vp), ("top_k_scalar", ctypes.c_int32),
        ("top_p", _vp), ("top_p_scalar", ctypes.c_float),
        ("min_p", _vp), ("min_p_scalar", ctypes.c_float),
        ("support_ids", _vp), ("support_width", ctypes.c_int32), ("support_ld", ctypes.c_int64),
        ("flags", ctypes.c_uint32), ("sample_seed", ctypes.c_uint64),
    ]


class ScoreOut(ctypes.Structure):
    _fields_ = [
        ("logprob_full", _vp), ("logprob_support", _vp), ("entropy_full", _vp),
        ("entropy_support", _vp), ("valid", _vp), ("status", _vp), ("support_size", _vp),
        ("support_mask", _vp), ("ctx", _vp), ("entropy_sum", _vp), ("valid_count", _vp),
        ("sampled", _vp),
    ]


class VsError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"libvs status {code}: {msg}")
        self.code = code


_lib = None


def load() -> ctypes.CDLL:
    """Load libvs.so (raises if it is missing: there is no fallback path)."""
    global _lib
    if _lib is None:
        if not LIB_PATH.exists():
            raise RuntimeError(f"{LIB_PATH} is missing: build it with sampling_support_b200.build")
        lib = ctypes.CDLL(str(LIB_PATH))
        i32, sz = ctypes.c_int32, ctypes.c_size_t
        lib.vs_score_fwd.argtypes = [ctypes.POINTER(ScoreArgs), ctypes.POINTER(ScoreOut), _vp, sz, _vp]
        lib.vs_score_fwd.restype = i32
        lib.vs_score_fwd_workspace_size.argtypes = [ctypes.POINTER(ScoreArgs)]
        lib.vs_score_fwd_workspace_size.restype = sz
        lib.vs_score_max_vocab.argtypes = [i32]
        lib.vs_score_max_vocab.restype = i32
        lib.vs_score_bwd.argtypes = [ctypes.POINTER(ScoreArgs), _vp, _vp, _vp, _vp, _vp, _vp, i32,
                                     ctypes.c_int64, i32, _vp]
        lib.vs_score_bwd.restype = i32
        lib.vs_l1_distance.argtypes = [i32, i32, ctypes.c_int64, i32, _vp, _vp, _vp, _vp, _vp, _vp,
                                       _vp, i32, ctypes.c_int64, _vp, sz, _vp]
        lib.vs_l1_distance.restype = i32
        lib.vs_l1_distance_sharded.argtypes = [i32, i32, ctypes.c_int64, i32, _vp, _vp, _vp, _vp,
                                               _vp, _vp, _vp, _vp, i32, ctypes.c_int64, _vp, sz,
                                               _vp]
        lib.vs_l1_distance_sharded.restype = i32
        lib.vs_l1_weight_sum.argtypes = [i32, _vp, _vp, _vp]
        lib.vs_l1_weight_sum.restype = i32
        lib.vs_l1_distance_workspace_size.argtypes = [i32]
        lib.vs_l1_distance_workspace_size.restype = sz
        lib.vs_fused_lmhead_score.argtypes = [i32, i32, i32, _vp, ctypes.c_int64, _vp,
                                              ctypes.c_int64, _vp, ctypes.c_float, _vp, i32,
                                              ctypes.c_float, ctypes.c_float, ctypes.c_uint32,
                                              ctypes.POINTER(ScoreOut), _vp, _vp, _vp, sz, _vp]
        lib.vs_fused_lmhead_score.restype = i32
        lib.vs_fused_lmhead_workspace_size.argtypes = [i32, i32, i32, i32]
        lib.vs_fused_lmhead_workspace_size.restype = sz
        lib.vs_fused_lmhead_bwd.argtypes = [i32, i32, i32, _vp, ctypes.c_int64, _vp,
                                            ctypes.c_int64, _vp, i32, _vp, _vp, _vp, _vp, _vp,
                                            _vp, _vp, ctypes.c_int64, _vp, ctypes.c_int64, _vp,
                                            sz, _vp]
        lib.vs_fused_lmhead_bwd.restype = i32
        lib.vs_fused_lmhead_bwd_workspace_size.argtypes = [i32, i32, i32]
        lib.vs_fused_lmhead_bwd_workspace_size.restype = sz
        lib.vs_fused_lmhead_partial_bytes.argtypes = [i32, i32]
        lib.vs_fused_lmhead_partial_bytes.restype = sz
        lib.vs_fused_lmhead_partial_workspace_size.argtypes = [i32, i32, i32, i32]
        lib.vs_fused_lmhead_partial_workspace_size.restype = sz
        lib.vs_fused_lmhead_partial.argtypes = [i32, i32, i32, i32, i32, _vp, ctypes.c_int64, _vp,
                                                ctypes.c_int64, _vp, ctypes.c_float, _vp, i32,
                                                _vp, _vp, sz, _vp]
        lib.vs_fused_lmhead_partial.restype = i32
        lib.vs_fused_lmhead_merge.argtypes = [i32, i32, i32, _vp, _vp, ctypes.c_float, _vp, i32,
                                              ctypes.c_float, ctypes.c_float, ctypes.c_uint32,
                                              ctypes.POINTER(ScoreOut), _vp, _vp, _vp]
        lib.vs_fused_lmhead_merge.restype = i32
        lib.vs_support_lmhead_score.argtypes = [i32, i32, i32, _vp, ctypes.c_int64, _vp,
                                                ctypes.c_int64, _vp, ctypes.c_float, _vp, _vp, i32,
                                                ctypes.c_int64, ctypes.c_uint32,
                                                ctypes.POINTER(ScoreOut), _vp, ctypes.c_int64, _vp]
        lib.vs_support_lmhead_score.restype = i32
        lib.vs_last_error.restype = ctypes.c_char_p
        lib.vs_version.restype = ctypes.c_char_p
        _lib = lib
    return _lib


def _check(rc: int) -> None:
    if rc != VS_OK:
        raise VsError(rc, load().vs_last_error().decode())


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return VS_BF16
    if t.dtype == torch.float32:
        return VS_F32
    raise TypeError(f"logits must be bfloat16 or float32, got {t.dtype}")


def _row_param(v, rows, dtype, device):
    """(tensor or None, scalar) for a per-row parameter."""
    if v is None:
        return None, None
    if isinstance(v, torch.Tensor):
        assert v.shape == (rows,) and v.dtype == dtype and v.device == device
        return v, 0
    return None, v


def make_args(logits, targets, temperature=1.0, top_k=0, top_p=1.0, min_p=0.0,
              support_ids=None, vocab=None, flags=0):
    rows, ld = logits.shape
    vocab = ld if vocab is None else vocab
    dev = logits.device
    a = ScoreArgs()
    a.rows, a.vocab, a.ld = rows, vocab, logits.stride(0)
    a.dtype = _dtype_code(logits)
    a.logits = logits.data_ptr()
    t_arr, t_s = _row_param(temperature, rows, torch.float32, dev)
    a.temperature = None if t_arr is None else t_arr.data_ptr()
    a.temperature_scalar = float(t_s if t_arr is None else 1.0)
    a.targets = targets.data_ptr()
    k_arr, k_s = _row_param(top_k, rows, torch.int32, dev)
    a.top_k = None if k_arr is None else k_arr.data_ptr()
    a.top_k_scalar = int(k_s if k_arr is None else 0)
    p_arr, p_s = _row_param(top_p, rows, torch.float32, dev)
    a.top_p = None if p_arr is None else p_arr.data_ptr()
    a.top_p_scalar = float(p_s if p_arr is None else 1.0)
    m_arr, m_s = _row_param(min_p, rows, torch.float32, dev)
    a.min_p = None if m_arr is None else m_arr.data_ptr()
    a.min_p_scalar = float(m_s if m_arr is None else 0.0)
    if support_ids is not None:
        a.support_ids = support_ids.data_ptr()
        a.support_width = support_ids.shape[1]
        a.support_ld = support_ids.stride(0)
    a.flags = flags
    keep = (logits, targets, t_arr, k_arr, p_arr, m_arr, support_ids)
    return a, keep


_SCORE_WS = {}


def score_workspace(nbytes, device):
    """A device workspace of at least nbytes, kept per device (vs_score_fwd
    needs no initial contents; calls on one stream may share it)."""
    if nbytes <= 0:
        return None
    key = (device.type, device.index)
    ws = _SCORE_WS.get(key)
    if ws is None or ws.numel() < nbytes:
        ws = torch.empty((nbytes + 15) // 16 * 16, dtype=torch.uint8, device=device)
        _SCORE_WS[key] = ws
    return ws


def score_fwd(logits, targets, temperature=1.0, top_k=0, top_p=1.0, min_p=0.0,
              support_ids=None, want_entropy=True, want_mask=False, want_grad=False,
              want_full=True, want_reduce=False, vocab=None, workspace=None, stream=None,
              sample_seed=None):
    """Run vs_score_fwd; returns a dict of device tensors.

    workspace: a uint8 device tensor of at least vs_score_fwd_workspace_size
    bytes (one call at a time); by default a buffer cached per device.
    sample_seed: when given, out["sampled"] holds one seeded Gumbel-max token
    per row drawn from its support."""
    lib = load()
    rows, ld = logits.shape
    vocab = ld if vocab is None else vocab
    dev = logits.device
    flags = (VS_WANT_ENTROPY if want_entropy else 0) | (VS_WANT_SUPPORT_MASK if want_mask else 0) \
        | (VS_WANT_GRAD if want_grad else 0) | (VS_WANT_SAMPLE if sample_seed is not None else 0)
    a, keep = make_args(logits, targets, temperature, top_k, top_p, min_p, support_ids, vocab, flags)
    if sample_seed is not None:
        a.sample_seed = int(sample_seed)
    f32 = dict(dtype=torch.float32, device=dev)
    out = {
        "lp_support": torch.empty(rows, **f32),
        "valid": torch.empty(rows, dtype=torch.uint8, device=dev),
        "status": torch.empty(rows, dtype=torch.int32, device=dev),
        "support_size": torch.empty(rows, dtype=torch.int32, device=dev),
    }
    if want_full:
        out["lp_full"] = torch.empty(rows, **f32)
    if want_entropy:
        out["h_support"] = torch.empty(rows, **f32)
        if want_full:
            out["h_full"] = torch.empty(rows, **f32)
    if want_mask:
        out["mask"] = torch.empty((rows, (vocab + 31) // 32), dtype=torch.int32, device=dev)
    if want_grad:
        out["ctx"] = torch.empty((rows, VS_CTX_BYTES_PER_ROW), dtype=torch.uint8, device=dev)
    if sample_seed is not None:
        out["sampled"] = torch.empty(rows, dtype=torch.int32, device=dev)
    if want_reduce:
        out["entropy_sum"] = torch.empty(1, dtype=torch.float64, device=dev)
        out["valid_count"] = torch.empty(1, dtype=torch.int32, device=dev)
    o = ScoreOut()
    o.logprob_full = _p(out.get("lp_full"))
    o.logprob_support = _p(out["lp_support"])
    o.entropy_full = _p(out.get("h_full"))
    o.entropy_support = _p(out.get("h_support"))
    o.valid = _p(out["valid"])
    o.status = _p(out["status"])
    o.support_size = _p(out["support_size"])
    o.support_mask = _p(out.get("mask"))
    o.ctx = _p(out.get("ctx"))
    o.entropy_sum = _p(out.get("entropy_sum") if want_entropy else None)
    o.valid_count = _p(out.get("valid_count"))
    o.sampled = _p(out.get("sampled"))
    if workspace is None:
        workspace = score_workspace(lib.vs_score_fwd_workspace_size(ctypes.byref(a)), dev)
    _check(lib.vs_score_fwd(ctypes.byref(a), ctypes.byref(o), _p(workspace),
                            0 if workspace is None else workspace.numel(), _stream(stream)))
    del keep
    return out


def score_bwd(logits, targets, ctx, g_lp_full=None, g_lp_support=None, g_h_full=None,
              g_h_support=None, temperature=1.0, top_k=0, top_p=1.0, min_p=0.0,
              support_ids=None, grad_dtype=torch.float32, mode=VS_GRAD_DENSE, out=None,
              vocab=None, stream=None):
    """Run vs_score_bwd; returns dlogits (dense [R, V] or sparse [R, W])."""
    lib = load()
    rows, ld = logits.shape
    vocab = ld if vocab is None else vocab
    a, keep = make_args(logits, targets, temperature, top_k, top_p, min_p, support_ids, vocab, 0)
    if out is None:
        if mode == VS_GRAD_SPARSE:
            out = torch.empty((rows, support_ids.shape[1]), dtype=torch.float32, device=logits.device)
        else:
            ld_g = (vocab + 7) // 8 * 8
            out = torch.empty((rows, ld_g), dtype=grad_dtype, device=logits.device)
    gcode = VS_BF16 if out.dtype == torch.bfloat16 else VS_F32
    _check(lib.vs_score_bwd(ctypes.byref(a), _p(ctx), _p(g_lp_full), _p(g_lp_support), _p(g_h_full),
                            _p(g_h_support), _p(out), gcode, out.stride(0), mode, _stream(stream)))
    del keep
    return out


def l1_distance(draft, target, row_weight=None, want_loss=True, want_grad=False,
                grad_dtype=torch.float32, workspace=None, vocab=None, stream=None,
                global_weight_sum=None):
    """vs_l1_distance; with global_weight_sum (a float64 device tensor of one
    element: the row-weight sum over every rank of a row-sharded batch)
    vs_l1_distance_sharded, whose gradient and loss value use that
    denominator."""
    lib = load()
    rows, ld = draft.shape
    vocab = ld if vocab is None else vocab
    dev = draft.device
    f32 = dict(dtype=torch.float32, device=dev)
    out = {"l1": torch.empty(rows, **f32), "accept": torch.empty(rows, **f32)}
    if want_loss:
        out["loss"] = torch.empty(3, **f32)
    if want_grad:
        out["grad"] = torch.empty((rows, ld), dtype=grad_dtype, device=dev)
    if workspace is None and (want_loss or want_grad):
        nbytes = lib.vs_l1_distance_workspace_size(rows)
        workspace = torch.empty((nbytes + 15) // 16 * 16, dtype=torch.uint8, device=dev)
    gcode = VS_BF16 if grad_dtype == torch.bfloat16 else VS_F32
    g = out.get("grad")
    common = (_p(out["l1"]), _p(out["accept"]), _p(out.get("loss")), _p(g), gcode,
              0 if g is None else g.stride(0), _p(workspace),
              0 if workspace is None else workspace.numel(), _stream(stream))
    if global_weight_sum is None:
        _check(lib.vs_l1_distance(rows, vocab, draft.stride(0), _dtype_code(draft), _p(draft),
                                  _p(target), _p(row_weight), *common))
    else:
        assert global_weight_sum.dtype == torch.float64 and global_weight_sum.device == dev
        _check(lib.vs_l1_distance_sharded(rows, vocab, draft.stride(0), _dtype_code(draft),
                                          _p(draft), _p(target), _p(row_weight),
                                          _p(global_weight_sum), *common))
    return out


def l1_weight_sum(rows, row_weight=None, out=None, device=None, stream=None):
    """vs_l1_weight_sum: this shard's weight sum as a float64 device tensor of
    one element (row_weight None: every row weighs 1)."""
    lib = load()
    dev = row_weight.device if row_weight is not None else (device or torch.device("cuda"))
    if out is None:
        out = torch.empty(1, dtype=torch.float64, device=dev)
    _check(lib.vs_l1_weight_sum(rows, _p(row_weight), _p(out), _stream(stream)))
    return out


def fused_lmhead_score(hidden, weight, targets, temperature, top_k, top_p, min_p,
                       want_entropy=True, want_grad=False, workspace=None, stream=None):
    """vs_fused_lmhead_score; want_grad also returns out["ctx"] (the saved
    state for fused_lmhead_bwd)."""
    lib = load()
    rows, hdim = hidden.shape
    vocab = weight.shape[0]
    dev = hidden.device
    f32 = dict(dtype=torch.float32, device=dev)
    out = {
        "lp_full": torch.empty(rows, **f32), "lp_support": torch.empty(rows, **f32),
        "valid": torch.empty(rows, dtype=torch.uint8, device=dev),
        "status": torch.empty(rows, dtype=torch.int32, device=dev),
        "support_size": torch.empty(rows, dtype=torch.int32, device=dev),
        "topk_ids": torch.empty((rows, top_k), dtype=torch.int32, device=dev),
        "topk_logprob": torch.empty((rows, top_k), **f32),
    }
    if want_entropy:
        out["h_full"] = torch.empty(rows, **f32)
        out["h_support"] = torch.empty(rows, **f32)
    if want_grad:
        out["ctx"] = torch.empty((rows, 64), dtype=torch.uint8, device=dev)
    o = ScoreOut()
    o.logprob_full = _p(out["lp_full"])
    o.logprob_support = _p(out["lp_support"])
    o.entropy_full = _p(out.get("h_full"))
    o.entropy_support = _p(out.get("h_support"))
    o.valid = _p(out["valid"])
    o.status = _p(out["status"])
    o.support_size = _p(out["support_size"])
    o.ctx = _p(out.get("ctx"))
    t_arr = temperature if isinstance(temperature, torch.Tensor) else None
    t_s = 1.0 if t_arr is not None else float(temperature)
    if workspace is None:
        nbytes = lib.vs_fused_lmhead_workspace_size(rows, vocab, hdim, top_k)
        workspace = torch.empty(max(16, (nbytes + 15) // 16 * 16), dtype=torch.uint8, device=dev)
    _check(lib.vs_fused_lmhead_score(rows, vocab, hdim, _p(hidden), hidden.stride(0), _p(weight),
                                     weight.stride(0), _p(t_arr), t_s, _p(targets), top_k,
                                     float(top_p), float(min_p),
                                     (VS_WANT_ENTROPY if want_entropy else 0)
                                     | (VS_WANT_GRAD if want_grad else 0), ctypes.byref(o),
                                     _p(out["topk_ids"]), _p(out["topk_logprob"]), _p(workspace),
                                     workspace.numel(), _stream(stream)))
    return out


def fused_lmhead_partial(hidden, weight_shard, vocab_begin, vocab_total, targets, temperature,
                         top_k, out=None, workspace=None, stream=None):
    """vs_fused_lmhead_partial: this shard's partial record block (a uint8
    device tensor of vs_fused_lmhead_partial_bytes(rows, top_k) bytes)."""
    lib = load()
    rows, hdim = hidden.shape
    count = weight_shard.shape[0]
    dev = hidden.device
    if out is None:
        out = torch.empty(lib.vs_fused_lmhead_partial_bytes(rows, top_k), dtype=torch.uint8,
                          device=dev)
    if workspace is None:
        nbytes = lib.vs_fused_lmhead_partial_workspace_size(rows, count, hdim, top_k)
        workspace = torch.empty(max(16, (nbytes + 15) // 16 * 16), dtype=torch.uint8, device=dev)
    t_arr = temperature if isinstance(temperature, torch.Tensor) else None
    t_s = 1.0 if t_arr is not None else float(temperature)
    _check(lib.vs_fused_lmhead_partial(rows, vocab_total, vocab_begin, count, hdim, _p(hidden),
                                       hidden.stride(0), _p(weight_shard), weight_shard.stride(0),
                                       _p(t_arr), t_s, _p(targets), top_k, _p(out),
                                       _p(workspace), workspace.numel(), _stream(stream)))
    return out


def fused_lmhead_merge(partials, rows, vocab_total, targets, temperature, top_k, top_p, min_p,
                       want_entropy=True, stream=None):
    """vs_fused_lmhead_merge over `partials` (uint8 [n_shards, block bytes],
    contiguous, the shards in vocabulary order); the outputs of
    fused_lmhead_score for the whole vocabulary."""
    lib = load()
    n_shards = partials.shape[0]
    dev = partials.device
    f32 = dict(dtype=torch.float32, device=dev)
    out = {
        "lp_full": torch.empty(rows, **f32), "lp_support": torch.empty(rows, **f32),
        "valid": torch.empty(rows, dtype=torch.uint8, device=dev),
        "status": torch.empty(rows, dtype=torch.int32, device=dev),
        "support_size": torch.empty(rows, dtype=torch.int32, device=dev),
        "topk_ids": torch.empty((rows, top_k), dtype=torch.int32, device=dev),
        "topk_logprob": torch.empty((rows, top_k), **f32),
    }
    if want_entropy:
        out["h_full"] = torch.empty(rows, **f32)
        out["h_support"] = torch.empty(rows, **f32)
    o = ScoreOut()
    o.logprob_full = _p(out["lp_full"])
    o.logprob_support = _p(out["lp_support"])
    o.entropy_full = _p(out.get("h_full"))
    o.entropy_support = _p(out.get("h_support"))
    o.valid = _p(out["valid"])
    o.status = _p(out["status"])
    o.support_size = _p(out["support_size"])
    t_arr = temperature if isinstance(temperature, torch.Tensor) else None
    t_s = 1.0 if t_arr is not None else float(temperature)
    _check(lib.vs_fused_lmhead_merge(rows, vocab_total, n_shards, _p(partials), _p(t_arr), t_s,
                                     _p(targets), top_k, float(top_p), float(min_p),
                                     VS_WANT_ENTROPY if want_entropy else 0, ctypes.byref(o),
                                     _p(out["topk_ids"]), _p(out["topk_logprob"]),
                                     _stream(stream)))
    return out


def fused_lmhead_bwd(hidden, weight, targets, top_k, fwd, g_lp_full=None, g_lp_support=None,
                     g_h_full=None, g_h_support=None, want_hidden=True, want_weight=True,
                     workspace=None, stream=None):
    """vs_fused_lmhead_bwd from a fused_lmhead_score(..., want_grad=True)
    result `fwd`; returns {"d_hidden": [rows, hidden] fp32, "d_weight":
    [vocab, hidden] fp32} (the requested ones)."""
    lib = load()
    rows, hdim = hidden.shape
    vocab = weight.shape[0]
    dev = hidden.device
    out = {}
    if want_hidden:
        out["d_hidden"] = torch.empty((rows, hdim), dtype=torch.float32, device=dev)
    if want_weight:
        out["d_weight"] = torch.empty((vocab, hdim), dtype=torch.float32, device=dev)
    if workspace is None:
        nbytes = lib.vs_fused_lmhead_bwd_workspace_size(rows, vocab, hdim)
        workspace = torch.empty(max(16, (nbytes + 15) // 16 * 16), dtype=torch.uint8, device=dev)
    dh, dw = out.get("d_hidden"), out.get("d_weight")
    _check(lib.vs_fused_lmhead_bwd(rows, vocab, hdim, _p(hidden), hidden.stride(0), _p(weight),
                                   weight.stride(0), _p(targets), top_k, _p(fwd["ctx"]),
                                   _p(fwd["topk_ids"]), _p(g_lp_full), _p(g_lp_support),
                                   _p(g_h_full), _p(g_h_support), _p(dh),
                                   0 if dh is None else dh.stride(0), _p(dw),
                                   0 if dw is None else dw.stride(0), _p(workspace),
                                   workspace.numel(), _stream(stream)))
    return out


def support_lmhead_score(hidden, weight, targets, temperature, support_ids, want_entropy=True,
                         want_logits=False, stream=None):
    """Support-only fused projection: z = hidden[i] . weight[s] / T_i for the
    kept ids s of each row's recorded support, then lp_S, H_S, valid, status
    and support size (no full-vocabulary quantity)."""
    lib = load()
    rows, hdim = hidden.shape
    vocab = weight.shape[0]
    width = support_ids.shape[1]
    dev = hidden.device
    f32 = dict(dtype=torch.float32, device=dev)
    out = {
        "lp_support": torch.empty(rows, **f32),
        "valid": torch.empty(rows, dtype=torch.uint8, device=dev),
        "status": torch.empty(rows, dtype=torch.int32, device=dev),
        "support_size": torch.empty(rows, dtype=torch.int32, device=dev),
    }
    if want_entropy:
        out["h_support"] = torch.empty(rows, **f32)
    if want_logits:
        out["support_logits"] = torch.empty((rows, width), **f32)
    o = ScoreOut()
    o.logprob_support = _p(out["lp_support"])
    o.entropy_support = _p(out.get("h_support"))
    o.valid = _p(out["valid"])
    o.status = _p(out["status"])
    o.support_size = _p(out["support_size"])
    t_arr = temperature if isinstance(temperature, torch.Tensor) else None
    t_s = 1.0 if t_arr is not None else float(temperature)
    lg = out.get("support_logits")
    _check(lib.vs_support_lmhead_score(rows, vocab, hdim, _p(hidden), hidden.stride(0), _p(weight),
                                       weight.stride(0), _p(t_arr), t_s, _p(targets),
                                       _p(support_ids), width, support_ids.stride(0),
                                       VS_WANT_ENTROPY if want_entropy else 0, ctypes.byref(o),
                                       _p(lg), lg.stride(0) if lg is not None else 0,
                                       _stream(stream)))
    return out
