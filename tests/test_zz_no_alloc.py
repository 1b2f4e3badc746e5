"""vs_l1_distance_static: the allocation-free variant of vs_l1_distance.

Some callers cannot call cudaMalloc (a plugin that cannot reach its host
application's device memory pool, or a serving loop that must not allocate
after start-up because cudaMalloc may synchronise the device).  For them the
library keeps the distance's scratch in a file-scope device array.  This test
calls the variant through the C ABI twice in a row, on different inputs, and
checks each result against vs_l1_distance with a caller workspace.  It lives
in its own file, collected last, and passes alone or after the other tests.
"""

import ctypes

import numpy as np
import pytest
import torch

import sampling_support_b200 as vsb
import workloads
from sampling_support_b200 import _binding as B

pytestmark = pytest.mark.gpu

STATIC_MAX_ROWS = 65536  # VS_L1_STATIC_MAX_ROWS


def _lib():
    lib = vsb.load()
    vp = ctypes.c_void_p
    lib.vs_l1_distance_static.argtypes = [ctypes.c_int32, ctypes.c_int32, ctypes.c_int64,
                                          ctypes.c_int32, vp, vp, vp, vp, vp, vp, vp,
                                          ctypes.c_int32, ctypes.c_int64, vp]
    lib.vs_l1_distance_static.restype = ctypes.c_int32
    return lib


def _dev(bits):
    return torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)


def _static_call(lib, d, t, w, grad_dtype):
    rows, ld = d.shape
    out = {"l1": torch.empty(rows, device="cuda"), "accept": torch.empty(rows, device="cuda"),
           "loss": torch.empty(3, device="cuda"),
           "grad": torch.empty((rows, ld), dtype=grad_dtype, device="cuda")}
    gcode = B.VS_BF16 if grad_dtype == torch.bfloat16 else B.VS_F32
    rc = lib.vs_l1_distance_static(
        rows, ld, ld, B.VS_BF16, d.data_ptr(), t.data_ptr(), w.data_ptr(),
        out["l1"].data_ptr(), out["accept"].data_ptr(), out["loss"].data_ptr(),
        out["grad"].data_ptr(), gcode, ld, torch.cuda.current_stream().cuda_stream)
    assert rc == B.VS_OK, lib.vs_last_error().decode()
    return out


def _close(a, b, rtol):
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    scale = np.maximum(np.abs(b), 1e-30)
    assert np.all(np.abs(a - b) <= rtol * scale), float((np.abs(a - b) / scale).max())


def test_static_scratch_matches_workspace_entry_point_twice():
    lib = _lib()
    cases = [workloads.distance(rows=96, vocab=40_000, seed=21),
             workloads.distance(rows=17, vocab=12_000, seed=22)]
    for w, gdt in zip(cases, [torch.float32, torch.bfloat16]):
        d, t = _dev(w["draft"]), _dev(w["target"])
        wt = torch.from_numpy(w["weight"]).cuda()
        got = _static_call(lib, d, t, wt, gdt)
        ref = vsb.l1_distance(d, t, wt, want_loss=True, want_grad=True, grad_dtype=gdt)
        torch.cuda.synchronize()
        _close(got["l1"], ref["l1"], 1e-4)
        _close(got["accept"], ref["accept"], 1e-4)
        _close(got["loss"], ref["loss"], 1e-4)
        g, r = got["grad"].double(), ref["grad"].double()
        rel = (g - r).norm(dim=1) / r.norm(dim=1).clamp_min(1e-30)
        assert rel.max().item() <= 2e-3


def test_static_scratch_rejects_rows_beyond_the_limit():
    lib = _lib()
    rows = STATIC_MAX_ROWS + 1
    rc = lib.vs_l1_distance_static(rows, 1024, 1024, B.VS_BF16, 16, 16, None, None, None, None,
                                   None, B.VS_F32, 0, None)
    assert rc == B.VS_ERR_UNSUPPORTED
    assert "VS_L1_STATIC_MAX_ROWS" in lib.vs_last_error().decode()
