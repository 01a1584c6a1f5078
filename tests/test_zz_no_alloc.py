"""bc_gemv_noalloc: the GEMV entry point that allocates nothing, for callers
that cannot give the library device memory (an operator inside another
framework whose allocator owns the device, or a serving path that must not
call cudaMalloc).  Its split-K scratch is a static device array.

The file is named to be collected last.  It passes alone in a fresh process
and after every other test: the first call on the device looks the array's
address up, and each call clears the tickets it uses."""
import numpy as np
import pytest
import torch

import activation_kv_sparsity_b200 as bc

DEV = "cuda:0"


def _inputs(d_in, d_out, k, seed):
    g = torch.Generator()
    g.manual_seed(seed)
    W = (torch.randn(d_in, d_out, generator=g) * 0.02).to(torch.bfloat16).to(DEV)
    x = torch.randn(d_in, generator=g).to(DEV)
    idx = None
    if k < d_in:
        idx = torch.sort(torch.randperm(d_in, generator=g)[:k])[0].to(torch.int32).to(DEV)
    return W, x, idx


@pytest.mark.gpu
@pytest.mark.parametrize("d_in,d_out,k", [(4096, 28672, 2048), (14336, 4096, 14336), (512, 768, 200),
                                          (14336, 256, 14336), (14336, 512, 7000)])
def test_noalloc_matches_gemv_twice(d_in, d_out, k):
    W, x, idx = _inputs(d_in, d_out, k, seed=d_out + k)
    scratch = torch.zeros(bc.bc_gemv_scratch_bytes(d_out), dtype=torch.uint8, device=DEV)
    ref = torch.empty(d_out, device=DEV)
    bc.gemv(W, x, idx, ref, scratch)
    for _ in range(2):                       # two calls in a row share the static scratch
        got = torch.full((d_out,), float("nan"), device=DEV)
        bc.gemv_noalloc(W, x, idx, got)
        torch.cuda.synchronize()
        # the same deterministic kernel with the same plan on the same inputs: bit for bit
        assert torch.equal(got, ref)
        assert np.isfinite(got.cpu().numpy()).all()


@pytest.mark.gpu
def test_noalloc_rejects_oversized_output():
    W = torch.zeros(1, dtype=torch.bfloat16, device=DEV)
    x = torch.zeros(4, device=DEV)
    y = torch.zeros(1, device=DEV)
    d_out = bc.bc_gemv_noalloc_max_dout() + 256
    st = bc.bc_gemv_noalloc(bc.C.c_void_p(W.data_ptr()), 4, d_out, bc.C.c_void_p(x.data_ptr()), None, 4,
                            bc.C.c_void_p(y.data_ptr()), None)
    assert st == bc.BC_EINVAL
    assert b"maximum" in bc.bc_last_error()
