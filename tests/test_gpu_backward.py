"""GPU backward pass (T = 1) against the float64 oracle's chain rule.

The oracle's backward is pinned by finite differences and by dense-attention
gradients (tests/test_oracle_backward.py).  The SIMT kernels compute in fp32
from the same input values; the tensor-core L side (bf16 rows of <= 128 keys)
multiplies bf16 operands into fp32.  The bar is max|g_gpu - g_oracle| <=
1e-4 max|g_oracle| for fp32 inputs, and 2e-2 max|g_oracle| for bf16 inputs,
where the gradients are rounded to bf16 on output (the forward pass's bars,
relative to the gradient's scale instead of V's).
"""
import numpy as np
import pytest
import torch

from oracle import monarch_attention_backward
from structured_sub_quadratic_b200.inputs import iid_qkv

pytestmark = pytest.mark.gpu

TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}

CASES = [
    # B, H, b1, b2, d, c1, c2
    (1, 2, 12, 10, 64, 1, 1),
    (2, 2, 9, 8, 64, 2, 2),
    (1, 1, 7, 9, 32, 3, 2),
    (1, 1, 5, 6, 24, 1, 2),
    (1, 2, 16, 16, 128, 1, 1),
    (1, 1, 30, 52, 128, 1, 1),
    (1, 1, 40, 40, 64, 2, 2),
]


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("B,H,b1,b2,d,c1,c2", CASES)
def test_backward_parity(cuda_lib, dtype, B, H, b1, b2, d, c1, c2):
    q, k, v = iid_qkv(B, H, b1 * b2, d, dtype, seed=b1 * 31 + b2)
    dO = iid_qkv(B, H, b1 * b2, d, dtype, seed=b1 * 31 + b2 + 1)[0]
    got = cuda_lib.monarch_attn_bwd(q.cuda(), k.cuda(), v.cuda(), dO.cuda(), b1, b2, 1, c1, c2)
    cuda_lib.check()
    assert cuda_lib.last_launches() > 0
    ref = monarch_attention_backward(*(x.double().numpy() for x in (q, k, v, dO)), b1, b2, c1, c2)
    for name, g, r in zip(("dq", "dk", "dv"), got, ref):
        g = g.double().cpu().numpy()
        assert np.isfinite(g).all(), name
        err, bound = np.abs(g - r).max(), TOL[dtype] * np.abs(r).max()
        assert err <= bound, f"{name}: max err {err:.3e} > {bound:.3e}"


def test_backward_is_deterministic(cuda_lib):
    q, k, v = (x.cuda() for x in iid_qkv(1, 2, 30 * 52, 128, torch.bfloat16, seed=4))
    dO = torch.randn_like(q)
    a = cuda_lib.monarch_attn_bwd(q, k, v, dO, 30, 52, 1)
    b = cuda_lib.monarch_attn_bwd(q, k, v, dO, 30, 52, 1)
    torch.cuda.synchronize()
    assert all(torch.equal(x, y) for x, y in zip(a, b))


TC_L_SIDE = [
    # B, H, b1, b2, d, c1, c2: bf16 rows of <= 128 keys, groups of <= 128 rows;
    # the untiled ones (c1 = c2 = 1, b2 <= 128) take the tensor-core R side too
    (1, 2, 90, 52, 128, 1, 1),   # the 480p latent's blocks
    (1, 2, 64, 64, 64, 1, 1),    # the 4K sweep's blocks
    (1, 1, 20, 128, 64, 1, 1),   # 128 positions per chunk
    (1, 1, 64, 20, 64, 1, 2),    # 128 keys per row, 64-key groups
    (1, 2, 100, 12, 128, 2, 1),  # 50-row groups
    (2, 1, 13, 11, 64, 3, 5),    # tiled, ragged groups
]


@pytest.mark.parametrize("B,H,b1,b2,d,c1,c2", TC_L_SIDE)
def test_backward_on_tensor_cores(cuda_lib, B, H, b1, b2, d, c1, c2):
    q, k, v = iid_qkv(B, H, b1 * b2, d, torch.bfloat16, seed=b1 * 7 + b2)
    dO = iid_qkv(B, H, b1 * b2, d, torch.bfloat16, seed=b1 * 7 + b2 + 1)[0]
    cuda_lib.timing_read()
    cuda_lib.timing_enable(True)
    try:
        got = cuda_lib.monarch_attn_bwd(q.cuda(), k.cuda(), v.cuda(), dO.cuda(), b1, b2, 1, c1, c2)
        names = set(cuda_lib.timing_read())
    finally:
        cuda_lib.timing_enable(False)
    cuda_lib.check()
    assert "bwd_tc_l_side" in names and "bwd_l_rows" not in names, names
    if c1 == 1 and c2 == 1:
        assert "bwd_tc_r_side" in names and "bwd_r_rows" not in names, names
    ref = monarch_attention_backward(*(x.double().numpy() for x in (q, k, v, dO)), b1, b2, c1, c2)
    for name, g, r in zip(("dq", "dk", "dv"), got, ref):
        g = g.double().cpu().numpy()
        assert np.isfinite(g).all(), name
        err, bound = np.abs(g - r).max(), TOL[torch.bfloat16] * np.abs(r).max()
        assert err <= bound, f"{name}: max err {err:.3e} > {bound:.3e}"
