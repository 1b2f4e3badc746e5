"""The C-ABI library loads, exports every function include/vs_api.h declares,
and rejects bad arguments on the host before touching the GPU (these calls
pass fake device addresses that are never dereferenced)."""

import ctypes
import re
from pathlib import Path

import pytest

import sampling_support_b200 as vsb
from sampling_support_b200 import _binding as B

HEADER = Path(__file__).resolve().parents[1] / "include" / "vs_api.h"


def declared_functions():
    text = HEADER.read_text()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(vs_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for want in ("vs_score_fwd", "vs_score_bwd", "vs_l1_distance", "vs_fused_lmhead_score",
                 "vs_last_error"):
        assert want in names


def test_library_exports_every_declared_symbol():
    lib = vsb.load()
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing
    assert lib.vs_version().decode().count(".") == 2


FAKE = 0x10000  # 16-byte aligned, never dereferenced by a rejected call


def _args(**kw):
    a = B.ScoreArgs()
    a.rows, a.vocab, a.ld, a.dtype = 4, 1000, 1000, B.VS_BF16
    a.logits, a.targets = FAKE, FAKE
    a.temperature_scalar, a.top_p_scalar, a.min_p_scalar, a.top_k_scalar = 1.0, 1.0, 0.0, 0
    for k, v in kw.items():
        setattr(a, k, v)
    return a


def _fwd(a, o=None):
    lib = vsb.load()
    o = o or B.ScoreOut()
    return lib.vs_score_fwd(ctypes.byref(a), ctypes.byref(o), None, 0, None)


@pytest.mark.parametrize("field,value", [
    ("rows", -1), ("vocab", 0), ("ld", 999), ("dtype", 7), ("logits", 0), ("logits", FAKE + 8),
    ("ld", 1001), ("targets", 0), ("temperature_scalar", 0.0),
    ("temperature_scalar", float("inf")), ("temperature_scalar", float("nan")),
    ("top_p_scalar", 0.0), ("top_p_scalar", 1.5), ("min_p_scalar", 1.0),
    ("min_p_scalar", -0.1),
])
def test_score_fwd_rejects_bad_arguments(field, value):
    lib = vsb.load()
    assert _fwd(_args(**{field: value})) == B.VS_ERR_INVALID_ARG
    assert lib.vs_last_error().decode() != ""


def test_score_fwd_rejects_flag_without_output():
    for flag in (B.VS_WANT_SUPPORT_MASK, B.VS_WANT_GRAD, B.VS_WANT_ENTROPY):
        assert _fwd(_args(flags=flag)) == B.VS_ERR_INVALID_ARG
    o = B.ScoreOut()
    o.entropy_support = FAKE  # entropy output without the entropy control
    assert _fwd(_args(), o) == B.VS_ERR_INVALID_ARG


def test_recorded_support_with_filter_is_rejected():
    a = _args(support_ids=FAKE, support_width=8, support_ld=8, top_p_scalar=0.9)
    assert _fwd(a) == B.VS_ERR_INVALID_ARG
    a = _args(support_ids=FAKE, support_width=B.VS_MAX_SUPPORT_WIDTH + 1,
              support_ld=B.VS_MAX_SUPPORT_WIDTH + 1)
    assert _fwd(a) == B.VS_ERR_UNSUPPORTED


def test_vocab_beyond_resident_limit_is_unsupported():
    lib = vsb.load()
    vmax = lib.vs_score_max_vocab(B.VS_BF16)
    assert vmax >= 151_936
    assert _fwd(_args(vocab=vmax + 8, ld=vmax + 8)) == B.VS_ERR_UNSUPPORTED


def test_zero_rows_is_a_no_op():
    assert _fwd(_args(rows=0, logits=0, targets=0)) == B.VS_OK


def test_score_bwd_rejects_bad_arguments():
    lib = vsb.load()
    a = _args()
    bad = [
        dict(ctx=0, dl=FAKE, ld=1000, mode=B.VS_GRAD_DENSE),
        dict(ctx=FAKE, dl=0, ld=1000, mode=B.VS_GRAD_DENSE),
        dict(ctx=FAKE, dl=FAKE, ld=999, mode=B.VS_GRAD_DENSE),
        dict(ctx=FAKE, dl=FAKE, ld=1000, mode=9),
        dict(ctx=FAKE, dl=FAKE, ld=1000, mode=B.VS_GRAD_SPARSE),  # needs a recorded support
    ]
    for b in bad:
        rc = lib.vs_score_bwd(ctypes.byref(a), b["ctx"], None, None, None, None, b["dl"],
                              B.VS_F32, b["ld"], b["mode"], None)
        assert rc == B.VS_ERR_INVALID_ARG, b


def test_l1_rejects_bad_arguments_and_small_workspace():
    lib = vsb.load()
    call = lib.vs_l1_distance
    assert call(4, 0, 8, B.VS_BF16, FAKE, FAKE, None, None, None, None, None, 0, 0, None, 0,
                None) == B.VS_ERR_INVALID_ARG
    assert call(4, 1000, 1000, B.VS_BF16, 0, FAKE, None, None, None, None, None, 0, 0, None, 0,
                None) == B.VS_ERR_INVALID_ARG
    need = lib.vs_l1_distance_workspace_size(4)
    assert need >= 4 * 8
    assert call(4, 1000, 1000, B.VS_BF16, FAKE, FAKE, None, None, None, FAKE, None, 0, 0, FAKE,
                need - 8, None) == B.VS_ERR_WORKSPACE


def test_score_fwd_workspace_size():
    """Computed supports and wide recorded lists need no scratch; narrow
    recorded lists (up to 64 ids) need the row list and one 20-byte partial
    per (row, chunk of 4,096 bf16 or 2,048 fp32 ids)."""
    lib = vsb.load()
    size = lambda a: lib.vs_score_fwd_workspace_size(ctypes.byref(a))
    assert size(_args()) == 0
    assert size(_args(rows=1 << 20, vocab=151_936, ld=151_936)) == 0
    assert size(_args(dtype=B.VS_F32)) == 0
    assert size(_args(support_ids=FAKE, support_width=65, support_ld=65)) == 0
    r16 = lambda n: (n + 15) // 16 * 16
    for rows, vocab, width, dt, chunk in [(4, 1000, 8, B.VS_BF16, 4096),
                                          (8192, 151_936, 64, B.VS_BF16, 4096),
                                          (3, 4097, 1, B.VS_BF16, 4096),
                                          (5, 151_936, 64, B.VS_F32, 2048)]:
        a = _args(rows=rows, vocab=vocab, ld=vocab + (-vocab) % 8, dtype=dt, support_ids=FAKE,
                  support_width=width, support_ld=width)
        nch = (vocab + chunk - 1) // chunk
        assert size(a) == 16 + 2 * r16(4 * rows) + r16(20 * rows * nch)


def _support_head(rows=4, vocab=1000, hidden=64, H=FAKE, ldh=64, W=FAKE, ldw=64, temp=1.0,
                  targets=FAKE, ids=FAKE, width=8, sld=8, flags=None, out=None, logits=None,
                  lld=0):
    lib = vsb.load()
    o = out if out is not None else B.ScoreOut()
    flags = B.VS_WANT_ENTROPY if flags is None else flags
    return lib.vs_support_lmhead_score(rows, vocab, hidden, H, ldh, W, ldw, None, temp, targets,
                                       ids, width, sld, flags, ctypes.byref(o), logits, lld, None)


def test_support_head_rejects_bad_arguments():
    inv, uns = B.VS_ERR_INVALID_ARG, B.VS_ERR_UNSUPPORTED
    assert _support_head(rows=-1) == inv
    assert _support_head(vocab=0) == inv
    assert _support_head(hidden=60, ldh=64, ldw=64) == uns      # not a multiple of 8
    assert _support_head(hidden=16392, ldh=16392, ldw=16392) == uns  # beyond 16384
    assert _support_head(width=B.VS_MAX_SUPPORT_WIDTH + 1, sld=2048) == uns
    assert _support_head(width=8, sld=7) == inv
    assert _support_head(temp=0.0) == inv
    assert _support_head(temp=float("nan")) == inv
    assert _support_head(H=FAKE + 8) == inv
    assert _support_head(ldh=60, hidden=56) == inv
    assert _support_head(ldh=56, hidden=64) == inv
    assert _support_head(targets=0) == inv
    assert _support_head(ids=0) == inv
    assert _support_head(flags=1 << 1) == inv                  # no mask on this path
    assert _support_head(logits=FAKE, lld=7) == inv
    for field in ("logprob_full", "entropy_full", "support_mask", "ctx", "sampled"):
        o = B.ScoreOut()
        setattr(o, field, FAKE)
        assert _support_head(out=o) == inv, field
    o = B.ScoreOut()
    o.entropy_support = FAKE
    assert _support_head(out=o, flags=0) == inv               # entropy needs VS_WANT_ENTROPY
    assert "not offered" in _last_error_after(lambda: _support_head(
        out=_with(B.ScoreOut(), "logprob_full", FAKE)))


def _with(o, field, value):
    setattr(o, field, value)
    return o


def _last_error_after(call):
    call()
    return vsb.load().vs_last_error().decode()


def test_support_head_zero_rows_is_a_no_op():
    assert _support_head(rows=0, H=0, W=0, targets=0, ids=0) == B.VS_OK


def test_sample_flag_and_output_go_together():
    lib = vsb.load()
    a = _args(flags=8)  # VS_WANT_SAMPLE without an output
    o = B.ScoreOut()
    assert lib.vs_score_fwd(ctypes.byref(a), ctypes.byref(o), FAKE, 1 << 20, None) == B.VS_ERR_INVALID_ARG
    a = _args()
    o = B.ScoreOut()
    o.sampled = FAKE  # an output without the flag
    assert lib.vs_score_fwd(ctypes.byref(a), ctypes.byref(o), FAKE, 1 << 20, None) == B.VS_ERR_INVALID_ARG


def test_fused_head_rejects_outputs_it_does_not_offer():
    lib = vsb.load()
    for field in ("sampled", "support_mask", "ctx"):
        o = B.ScoreOut()
        setattr(o, field, FAKE)
        rc = lib.vs_fused_lmhead_score(4, 1000, 64, FAKE, 64, FAKE, 64, None, 1.0, FAKE, 8, 1.0, 0.0,
                                       0, ctypes.byref(o), None, None, FAKE, 1 << 30, None)
        assert rc == B.VS_ERR_INVALID_ARG, field
    o = B.ScoreOut()
    rc = lib.vs_fused_lmhead_score(4, 1000, 64, FAKE, 64, FAKE, 64, None, 1.0, FAKE, 8, 1.0, 0.0,
                                   8, ctypes.byref(o), None, None, FAKE, 1 << 30, None)
    assert rc == B.VS_ERR_INVALID_ARG  # VS_WANT_SAMPLE
