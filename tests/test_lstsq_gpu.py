"""GPU regularised least squares with a cached factorisation against the fp64 oracle (the
MOD-DiT page, Method section, Stage 1: (M^T M + lambda I) X = M^T S_t, factored once and
reused across heads and steps)."""
import numpy as np
import pytest
import torch

import oracle
import video_dit_sparse_dsa_b200 as dsa

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("m,p,batch,lam", [(5000, 3, 24, 1e-2), (90000, 3, 48, 1e-3), (20000, 17, 7, 0.5),
                                           (33, 32, 2, 1.0)])
def test_lstsq_against_oracle(m, p, batch, lam):
    g = torch.Generator().manual_seed(m + p)
    M = torch.randn((m, p), generator=g, dtype=torch.float32)
    S = torch.randn((batch, m), generator=g, dtype=torch.float32)
    Mc, Sc = M.cuda(), S.cuda()
    L = dsa.lstsq_factor(Mc, lam)
    X = dsa.lstsq_solve(Mc, L, Sc)
    assert dsa.device_status()[0] == 0
    ref = oracle.lstsq(M.double(), lam, S.double())
    got = X.cpu().numpy()
    # fp32 inputs and outputs, fp64 sums: the result is the exact solution rounded to fp32
    np.testing.assert_allclose(got, ref, rtol=1e-5, atol=1e-6 * np.abs(ref).max())
    # the factor is the Cholesky factor of M^T M + lambda I
    G = M.double().numpy().T @ M.double().numpy() + lam * np.eye(p)
    Lh = L.cpu().numpy()
    np.testing.assert_allclose(Lh @ Lh.T, G, rtol=1e-12, atol=1e-9 * np.abs(G).max())
    assert np.all(np.triu(Lh, 1) == 0.0)


def test_lstsq_factor_reused_across_batches():
    g = torch.Generator().manual_seed(3)
    M = torch.randn((4000, 5), generator=g).cuda()
    L = dsa.lstsq_factor(M, 0.1)
    for seed in range(3):
        S = torch.randn((10, 4000), generator=torch.Generator().manual_seed(seed)).cuda()
        X = dsa.lstsq_solve(M, L, S)
        np.testing.assert_allclose(X.cpu().numpy(), oracle.lstsq(M.cpu().double(), 0.1, S.cpu().double()),
                                   rtol=1e-5, atol=1e-6)
    assert dsa.device_status()[0] == 0


def test_singular_system_is_reported():
    """lambda = 0 with a rank-deficient M: the factorisation records a device error."""
    M = torch.zeros((100, 3), device="cuda")
    M[:, 0] = 1.0
    dsa.lstsq_factor(M, 0.0)
    st, site, _ = dsa.device_status()
    assert st == 6 and site == 95


def test_lstsq_solve_is_one_launch_without_workspace_and_reproducible():
    """The solve takes no workspace (a null pointer is accepted) and, summing in a fixed order,
    gives the same bits on every call."""
    import ctypes

    lib = dsa.load_library()
    assert lib.dsa_lstsq_workspace_size(90000, 3, 24) == 0
    g = torch.Generator().manual_seed(5)
    M = torch.rand((90000, 3), generator=g).cuda()
    S = torch.rand((24, 90000), generator=g).cuda()
    L = dsa.lstsq_factor(M, 1e-3)
    X = torch.empty((24, 3), dtype=torch.float32, device="cuda")
    st = lib.dsa_lstsq_solve(90000, 3, 24, ctypes.c_void_p(M.data_ptr()), ctypes.c_void_p(L.data_ptr()),
                             ctypes.c_void_p(S.data_ptr()), ctypes.c_void_p(X.data_ptr()), None, 0,
                             ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0
    again = dsa.lstsq_solve(M, L, S)
    torch.cuda.synchronize()
    assert torch.equal(X, again)
    ref = oracle.lstsq(M.cpu().double(), 1e-3, S.cpu().double())
    np.testing.assert_allclose(X.cpu().numpy(), ref, rtol=1e-5, atol=1e-6 * np.abs(ref).max())
