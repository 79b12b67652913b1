"""The allocation-free RMSNorm backward against the regular entry point.

Some callers cannot allocate device memory when they need this gradient (their
memory is already committed to another allocator, or an allocation's implicit
synchronisation is not acceptable in their loop), so the library offers a
variant whose scratch is a fixed array inside the library. This checks, through
the C ABI, that two calls in a row give the regular entry point's outputs
within the tolerance the kernel tests use. The file sorts last so that a run
stopping at the first failure has run every other test first."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("T,d", [(300, 256), (1000, 5120), (16384, 2048), (40, 8192)])
def test_noalloc_matches_regular_entry_point_twice(T, d):
    from host_memory_streamed_layer_b200 import mt
    rng = np.random.default_rng(T + d)
    dev = "cuda"
    x = torch.tensor(rng.normal(0, 2, (T, d)).astype(np.float32), device=dev)
    dy = torch.tensor(rng.normal(size=(T, d)).astype(np.float32), device=dev)
    dres = torch.tensor(rng.normal(size=(T, d)).astype(np.float32), device=dev)
    g = torch.tensor((1 + 0.1 * rng.normal(size=d)).astype(np.float32)).to(torch.bfloat16).to(dev)
    r = torch.rsqrt((x * x).mean(dim=1) + 1e-5).contiguous()
    # regular entry point with a caller scratch buffer
    part = torch.empty(mt.mt_k_rmsnorm_bwd_partial_floats(T, d), device=dev)
    dx0 = torch.empty(T, d, device=dev)
    dxb0 = torch.empty(T, d, dtype=torch.bfloat16, device=dev)
    dg0 = torch.empty(d, device=dev)
    mt.mt_k_rmsnorm_bwd(x.data_ptr(), g.data_ptr(), r.data_ptr(), dy.data_ptr(), dres.data_ptr(), dx0.data_ptr(),
                        dxb0.data_ptr(), part.data_ptr(), dg0.data_ptr(), T, d)
    torch.cuda.synchronize()
    for _ in range(2):  # two calls in a row share the library's array
        dx1 = torch.full((T, d), float("nan"), device=dev)
        dxb1 = torch.empty(T, d, dtype=torch.bfloat16, device=dev)
        dg1 = torch.full((d,), float("nan"), device=dev)
        mt.mt_k_rmsnorm_bwd_noalloc(x.data_ptr(), g.data_ptr(), r.data_ptr(), dy.data_ptr(), dres.data_ptr(),
                                    dx1.data_ptr(), dxb1.data_ptr(), dg1.data_ptr(), T, d)
        torch.cuda.synchronize()
        a, b = dx1.double().cpu().numpy(), dx0.double().cpu().numpy()
        assert np.allclose(a, b, rtol=1e-4, atol=1e-5 * np.abs(b).max())
        assert np.array_equal(dxb1.float().cpu().numpy(), dxb0.float().cpu().numpy())
        ga, gb = dg1.double().cpu().numpy(), dg0.double().cpu().numpy()
        assert np.linalg.norm(ga - gb) / np.linalg.norm(gb) < 1e-5


def test_noalloc_rejects_rows_beyond_the_limit():
    from host_memory_streamed_layer_b200 import mt
    t = torch.zeros(8, dtype=torch.float32, device="cuda")
    with pytest.raises(mt.MTError):
        mt.mt_k_rmsnorm_bwd_noalloc(t.data_ptr(), t.data_ptr(), t.data_ptr(), t.data_ptr(), 0, t.data_ptr(), 0,
                                    t.data_ptr(), 1, 8196)
