"""The linear-state entry point that allocates nothing.

Some callers cannot allocate device memory when they run the layer (their
device memory is reserved by another allocator, or an allocation's implicit
synchronisation is not allowed in their loop).  zb_linear_state_static serves
them with a fixed scratch array inside the library instead of a caller
workspace.  This test calls it through the C ABI twice in a row, with
different shapes (the scratch keeps the previous call's contents), and checks
each result against the workspace entry point zb_linear_state (the same
kernels on the same grid, so bit for bit) and against the fp64 oracle (at the
bar of the other linear-state tests).  It lives in a file of its own that
pytest collects last.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth
from tests.gpu_helpers import host, rel_err_per_head, sync_ok, workload

pytestmark = pytest.mark.gpu


def _lib():
    from linear_hybrid_attention_b200 import _lib
    lib = _lib.load()
    fn = lib.zb_linear_state_static
    fn.restype = ctypes.c_int32
    fn.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_int32,
                   ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    lib.zb_linear_state_static_scratch_bytes.restype = ctypes.c_size_t
    return lib


def test_static_scratch_state_matches_workspace_entry_point():
    import linear_hybrid_attention_b200 as zb
    lib = _lib()
    assert lib.zb_linear_state_static_scratch_bytes() == 8 << 20
    # two calls in a row: a larger grid first, then a smaller one
    for call, (heads, n, seed) in enumerate([(16, 43968, 21), (3, 5000, 22)]):
        w = workload("linear256", heads=heads, n_tokens=n)
        _, K, V = synth.make_qkv(w, device="cuda", seed=seed)
        S_ref, z_ref = zb.zb_linear_state(K, V)
        S = torch.full((heads, 64, 64), float("nan"), dtype=torch.float32, device="cuda")
        z = torch.full((heads, 64), float("nan"), dtype=torch.float32, device="cuda")
        st = lib.zb_linear_state_static(K.data_ptr(), V.data_ptr(), heads, n, 64, S.data_ptr(),
                                        z.data_ptr(), torch.cuda.current_stream().cuda_stream)
        assert st == 0, f"call {call}: status {st}"
        sync_ok()
        # same kernels, same grid, fixed-order reduction: identical bits
        assert torch.equal(S, S_ref) and torch.equal(z, z_ref), f"call {call}"
        S64, z64 = oracle.linear_state(host(K), host(V))
        assert rel_err_per_head(S.cpu().numpy(), S64) <= 1e-2
        np.testing.assert_allclose(z.cpu().numpy(), z64, rtol=5e-3)


def test_static_scratch_rejects_shapes_beyond_its_size():
    lib = _lib()
    # 600 heads need more partial-state scratch than the fixed 8 MiB: refused, nothing launched
    assert lib.zb_linear_state_static(0x10000, 0x10000, 600, 1000, 64, 0x10000, 0x10000, None) == 4
