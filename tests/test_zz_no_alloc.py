"""mt_rmsnorm_bwd_noalloc: the RMSNorm backward without a caller workspace.

Some callers cannot allocate device memory for a workspace: their device
memory is owned and budgeted by another allocator (a framework's caching
pool, a budget fixed at start-up) and they have no spare buffer to hand over.
For them the library keeps a fixed scratch array of its own. This test calls
the entry point through the C ABI twice in a row and checks both results
against the workspace entry point, mt_rmsnorm_bwd, on the same inputs. It
lives in its own file, collected last, and passes alone in a fresh process
as well as after the other tests.
"""
import numpy as np
import pytest

from host_offloaded_layer_b200 import _lib as L
from host_offloaded_layer_b200 import synth

pytestmark = pytest.mark.gpu

TOL = 2e-2  # the relative Frobenius tolerance of the other parity tests


def _rel(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def _f64(t):
    import torch
    if t.dtype == torch.bfloat16:
        return synth.bf16_bits_to_f32(t.view(torch.int16).cpu().numpy().view(np.uint16)).astype(np.float64)
    return t.cpu().numpy().astype(np.float64)


def _dev(bits):
    import torch
    return torch.from_numpy(bits.view(np.int16).copy()).cuda().view(torch.bfloat16)


def test_noalloc_rmsnorm_bwd_matches_workspace_entry_point_twice():
    import torch
    for call, (rows, H) in enumerate(((1000, 3584), (4097, 512))):  # two calls in a row, different shapes
        def bits(tid, n, std=1.0):
            return synth.f32_to_bf16_bits(synth.normal_f32(77, call, tid, n, std))
        x, dy, dres = _dev(bits(1, rows * H)), _dev(bits(2, rows * H)), _dev(bits(3, rows * H))
        g = _dev(synth.f32_to_bf16_bits((1.0 + synth.normal_f32(77, call, 4, H, 0.2)).astype(np.float32)))
        y = torch.empty_like(x)
        rstd = torch.empty(rows, dtype=torch.float32, device="cuda")
        L.mt_rmsnorm_fwd(x, g, y, rstd, rows, H, 1e-6)
        # the existing entry point, with a caller workspace
        nws = L.mt_rmsnorm_bwd_workspace_bytes(rows, H)
        ws = torch.empty(nws, dtype=torch.uint8, device="cuda")
        dx_ref = torch.empty_like(x)
        dg_ref = torch.empty(H, dtype=torch.float32, device="cuda")
        L.mt_rmsnorm_bwd(dy, x, g, rstd, dres, dx_ref, dg_ref, rows, H, ws, nws)
        # the entry point without one
        dx = torch.full_like(x, float("nan"))
        dg = torch.full((H,), float("nan"), dtype=torch.float32, device="cuda")
        L.mt_rmsnorm_bwd_noalloc(dy, x, g, rstd, dres, dx, dg, rows, H)
        torch.cuda.synchronize()
        assert _rel(_f64(dx), _f64(dx_ref)) <= TOL
        assert _rel(_f64(dg), _f64(dg_ref)) <= TOL
        assert torch.equal(dx.view(torch.int16), dx_ref.view(torch.int16))
        assert torch.equal(dg, dg_ref)


def test_noalloc_at_its_exact_limit_matches_workspace_entry_point():
    """ceil(rows / 64) * H = 2,097,152 exactly (16384 rows of 8192): the largest call the
    fixed scratch takes, bit for bit equal to the workspace entry point."""
    import torch
    rows, H = 16384, 8192

    def bits(tid, n, std=1.0):
        return synth.f32_to_bf16_bits(synth.normal_f32(78, 0, tid, n, std))
    x, dy = _dev(bits(1, rows * H)), _dev(bits(2, rows * H))
    g = _dev(synth.f32_to_bf16_bits((1.0 + synth.normal_f32(78, 0, 4, H, 0.2)).astype(np.float32)))
    y = torch.empty_like(x)
    rstd = torch.empty(rows, dtype=torch.float32, device="cuda")
    L.mt_rmsnorm_fwd(x, g, y, rstd, rows, H, 1e-6)
    del y
    nws = L.mt_rmsnorm_bwd_workspace_bytes(rows, H)
    assert nws == 8 << 20  # the scratch array's size
    ws = torch.empty(nws, dtype=torch.uint8, device="cuda")
    dx_ref = torch.empty_like(x)
    dg_ref = torch.empty(H, dtype=torch.float32, device="cuda")
    L.mt_rmsnorm_bwd(dy, x, g, rstd, None, dx_ref, dg_ref, rows, H, ws, nws)
    dx = torch.full_like(x, float("nan"))
    dg = torch.full((H,), float("nan"), dtype=torch.float32, device="cuda")
    L.mt_rmsnorm_bwd_noalloc(dy, x, g, rstd, None, dx, dg, rows, H)
    torch.cuda.synchronize()
    assert L.mt_device_error(clear=True) == 0
    assert torch.equal(dx.view(torch.int16), dx_ref.view(torch.int16))
    assert torch.equal(dg, dg_ref)


@pytest.mark.parametrize("rows,H", [(16385, 8192), (64 * 600, 8192)])  # one row past the limit, and far past it
def test_noalloc_rejects_sizes_beyond_its_scratch_and_writes_nothing(rows, H):
    import torch
    x = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    r = torch.zeros(16, dtype=torch.float32, device="cuda")
    dx = torch.full((16,), 3.0, dtype=torch.bfloat16, device="cuda")
    dg = torch.full((16,), 5.0, dtype=torch.float32, device="cuda")
    with pytest.raises(L.MTError) as e:
        L.mt_rmsnorm_bwd_noalloc(x, x, x, r, None, dx, dg, rows, H)
    assert e.value.name == "MT_ERR_WORKSPACE"
    assert "scratch" in str(e.value)
    torch.cuda.synchronize()
    assert torch.all(dx == 3.0) and torch.all(dg == 5.0), "a rejected call wrote its outputs"
