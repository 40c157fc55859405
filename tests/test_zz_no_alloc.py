"""The allocation-free Mamba-1 backward (msc_selective_scan_bwd_static).

For callers that may not allocate device memory when they run the backward
pass, the library offers an entry point whose scratch is a fixed array in the
library's own device memory.  This test calls it through the C ABI twice in a
row and checks both results against the workspace entry point
(msc_selective_scan_bwd) on the same inputs.  Both run the same kernels in
the same fixed summation order, so the results must be equal bit for bit;
the cases cover one launch (16 states) and the slab layout (200 states, four
launches whose token sums cross the slabs through the scratch).  It also
checks that sizes beyond the array are refused on the host.  It sits in a file that pytest collects last, so that a run stopping
at the first failure has already run every other test.
"""
import ctypes

import pytest

from selective_state_space_14_b200 import workloads as W
from tests._util import dev, m1_device_args

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def msc():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from selective_state_space_14_b200 import msc as m
    m.lib()
    return m


@pytest.mark.parametrize("io,N,L", [("f32", 16, 700), ("bf16", 16, 700), ("bf16", 200, 333)])
def test_static_scratch_backward_matches_workspace_backward(msc, io, N, L):
    p = W.m1_problem(2, 96, N, L, io=io, seed=2024, bias=True, with_h0=True)
    assert msc.msc_selective_scan_bwd_workspace_bytes(2, 96, N, L, 1) <= \
        msc.MSC_STATIC_SCRATCH_BYTES
    a = m1_device_args(p)
    dout = dev(p.dout)
    _, _, saved = msc.msc_selective_scan_fwd(**a)
    ref = msc.msc_selective_scan_bwd(saved_states=saved, dout=dout, **a)
    torch.cuda.synchronize()
    ref = {k: v.clone() for k, v in ref.items() if v is not None}
    for call in range(2):  # two calls in a row share the static array
        got = msc.msc_selective_scan_bwd_static(saved_states=saved, dout=dout, **a)
        torch.cuda.synchronize()
        for k, v in ref.items():
            assert torch.equal(got[k], v), f"{k} (call {call}) differs from the workspace backward"


def test_static_scratch_rejects_oversize(msc):
    """Sizes whose scratch exceeds the static array are refused on the host
    (MSC_ERR_WORKSPACE, nothing launched); the size check comes before any
    pointer is used, so the arguments carry no device buffers."""
    Bsz, Dm, N, L, G = 64, 4096, 16, 4096, 1
    need = msc.msc_selective_scan_bwd_workspace_bytes(Bsz, Dm, N, L, G)
    assert need > msc.MSC_STATIC_SCRATCH_BYTES
    a = msc.SsBwdArgs()
    a.struct_size = ctypes.sizeof(msc.SsBwdArgs)
    a.io_dtype, a.batch, a.dim, a.dstate, a.seqlen, a.ngroups = msc.MSC_BF16, Bsz, Dm, N, L, G
    a.delta_softplus = 1
    st = msc.lib().msc_selective_scan_bwd_static(ctypes.byref(a), None)
    assert st == 5  # MSC_ERR_WORKSPACE
    err = msc.lib().msc_last_error().decode()
    assert "static scratch" in err and str(need) in err
