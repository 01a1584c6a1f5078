"""Single-kernel parity on the GPU: the column-gathered GEMV, the exact
top-k selection and the split-K attention, each through the C ABI, against
the oracle on the same seeded inputs."""
import math

import numpy as np
import pytest
import torch

import activation_kv_sparsity_b200 as bc
from oracle import decoder as od
from parity import bits, pool_from_tokens

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _gen(seed):
    g = torch.Generator()
    g.manual_seed(seed)
    return g


@pytest.mark.parametrize("d_in,d_out", [(512, 768), (512, 3584), (1792, 512), (4096, 6144), (4096, 4096),
                                        (14336, 4096), (4096, 28672), (14336, 256), (4096, 512), (40, 256)])
def test_gemv_dense_and_gathered(d_in, d_out):
    g = _gen(d_in * 7 + d_out)
    W = (torch.randn(d_in, d_out, generator=g) * 0.02).to(torch.bfloat16)
    x = torch.randn(d_in, generator=g)
    Wd, xd = W.to(DEV), x.to(DEV)
    scratch = torch.zeros(bc.bc_gemv_scratch_bytes(d_out), dtype=torch.uint8, device=DEV)
    wb = bits(W)
    x64 = x.double().numpy()
    absmag = np.abs(x64) @ np.abs(od.bf16_to_f64(wb))     # summation error scale
    for k in sorted({None, 1, 37, d_in // 2 + 3, d_in} - {None}) + [None]:
        if k is not None and k > d_in:
            continue
        if k is None:
            idx = None
            rows = None
        else:
            rows = np.sort(torch.randperm(d_in, generator=g)[:k].numpy())
            idx = torch.from_numpy(rows.astype(np.int32)).to(DEV)
        y = torch.full((d_out,), float("nan"), device=DEV)
        bc.gemv(Wd, xd, idx, y, scratch)
        torch.cuda.synchronize()
        ref = od.gemv_rows(x64, wb, rows)
        err = np.abs(y.cpu().double().numpy() - ref)
        mag = absmag if rows is None else np.abs(x64[rows]) @ np.abs(od.bf16_to_f64(wb[rows]))
        assert (err <= 1e-5 * mag + 1e-30).all(), (k, float((err / (mag + 1e-30)).max()))


def test_gemv_is_deterministic():
    g = _gen(5)
    W = (torch.randn(14336, 4096, generator=g) * 0.02).to(torch.bfloat16).to(DEV)
    x = torch.randn(14336, generator=g).to(DEV)
    scratch = torch.zeros(bc.bc_gemv_scratch_bytes(4096), dtype=torch.uint8, device=DEV)
    ys = []
    for _ in range(3):
        y = torch.empty(4096, device=DEV)
        bc.gemv(W, x, None, y, scratch)
        ys.append(y.clone())
    assert torch.equal(ys[0], ys[1]) and torch.equal(ys[1], ys[2])


@pytest.mark.parametrize("n", [1, 7, 100, 1024, 1792, 4096, 14336, 16384])
def test_select_topk_exact(n):
    g = _gen(n)
    for trial in range(4):
        v = torch.randn(n, generator=g)
        if trial == 1:
            v = torch.round(v * 4) / 4            # many ties
        if trial == 2:
            v = torch.zeros(n)                    # all tied
            v[:: 3] = 1.0
        if trial == 3:
            v = 1.0 + 1e-4 * v                    # narrow range: crowded bins
        vd = v.to(DEV)
        for k in sorted({1, max(1, n // 3), max(1, math.ceil(0.7 * n - 1e-9)), n}):
            idx = torch.full((k,), -1, dtype=torch.int32, device=DEV)
            bc.select_topk(vd, k, idx)
            torch.cuda.synchronize()
            want = od.channel_select(v.double().numpy(), 1.0, k=k)
            np.testing.assert_array_equal(idx.cpu().numpy(), want, err_msg=f"n={n} k={k} trial={trial}")


@pytest.mark.parametrize("hd", [64, 128])
@pytest.mark.parametrize("n_tok", [1, 16, 17, 200, 2049, 40000])
def test_attention_over_page_lists(hd, n_tok):
    g = _gen(n_tok + hd)
    Hkv, G = 2 if hd == 64 else 8, 4
    n_keep = n_tok
    k = (torch.randn(Hkv, n_tok, hd, generator=g) * 2).to(torch.bfloat16)
    v = torch.randn(Hkv, n_tok, hd, generator=g).to(torch.bfloat16)
    q = torch.randn(Hkv * G, hd, generator=g)
    P = -(-n_tok // 16)
    Pmax = P + 3
    pool = pool_from_tokens(k.to(DEV), v.to(DEV), Pmax)
    qd = q.to(DEV)
    scratch = torch.zeros(bc.bc_attention_scratch_bytes(Hkv * G, hd), dtype=torch.uint8, device=DEV)
    kf, vf = od.bf16_to_f64(bits(k)), od.bf16_to_f64(bits(v))
    q64 = q.double().numpy()
    # dense list, then a sparse list per head (always with the last page)
    lists = [None]
    if P > 2:
        sel = []
        for h in range(Hkv):
            s = torch.randperm(P - 1, generator=g)[: max(1, (P - 1) // 3)].numpy()
            sel.append(np.sort(np.append(s, P - 1)))
        lists.append(sel)
    for sel in lists:
        out = torch.full((Hkv * G, hd), float("nan"), device=DEV)
        if sel is None:
            bc.attention(qd, pool, Hkv, G, hd, Pmax, None, P, n_tok, out, scratch)
        else:
            K = len(sel[0])
            pages = torch.zeros(Hkv, Pmax, dtype=torch.int32)
            for h in range(Hkv):
                pages[h, :K] = torch.from_numpy(sel[h].astype(np.int32))
            bc.attention(qd, pool, Hkv, G, hd, Pmax, pages.to(DEV), K, n_tok, out, scratch)
        torch.cuda.synchronize()
        got = out.cpu().double().numpy()
        for h in range(Hkv):
            if sel is None:
                tok = np.arange(n_tok)
            else:
                tok = np.concatenate([np.arange(p * 16, min(p * 16 + 16, n_tok)) for p in sel[h]])
            ref = od.attention(q64[h * G:(h + 1) * G], kf[h], vf[h], tok)
            err = np.abs(got[h * G:(h + 1) * G] - ref).max() / np.abs(ref).max()
            assert err < 1e-4, (h, err)
