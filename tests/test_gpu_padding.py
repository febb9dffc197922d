"""GPU parity with padding (N_real < b1 * b2) against the float64 oracle.

Reading (the pages give only m = ceil(N / b) and pre-padding for ViT's
N = 197): the objective covers the real tokens; pad keys get zero R weight,
a column group without a real key zero L weight, pad query rows are left out.
Each case below drives one kernel path through its masks:
  * ViT-B's 197 tokens as 15 x 14 with 13 pad tokens first, T = 3: the
    one-CTA-per-head kernel (bf16) and the SIMT kernels (fp32);
  * a post-padded 480p-like head: paired tcgen05 R tiles;
  * 80-position chunks in two column groups, 45 pad tokens first (chunk 0's
    first group holds no real key): unpaired tcgen05 R tiles;
  * 100-key column groups with a whole pad chunk: the streaming R kernel;
  * 400 keys per L row whose first 68 are masked: the online output kernel
    starting on a key tile with no real key;
  * T = 2 (later steps on the SIMT kernels), T = 0, odd d, one real token.
Bar: 1e-4 max|V| (fp32) and 2e-2 max|V| (bf16), max over the real values.
"""
import numpy as np
import pytest
import torch

from oracle import monarch_attention
from structured_sub_quadratic_b200.inputs import iid_qkv

pytestmark = pytest.mark.gpu

TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}

CASES = [
    # B, H, n_real, b1, b2, pad_front, d, T, c1, c2, dtype
    (4, 12, 197, 15, 14, True, 64, 3, 1, 1, torch.bfloat16),
    (2, 3, 197, 15, 14, True, 64, 3, 1, 1, torch.float32),
    (1, 2, 197, 15, 14, False, 64, 3, 1, 1, torch.bfloat16),
    (1, 2, 4680 - 37, 90, 52, False, 128, 1, 1, 1, torch.bfloat16),
    (1, 2, 4680 - 37, 90, 52, True, 128, 1, 1, 1, torch.bfloat16),
    (1, 2, 40 * 80 - 45, 40, 80, True, 128, 1, 2, 2, torch.bfloat16),
    (1, 2, 12 * 100 - 150, 12, 100, True, 64, 1, 1, 1, torch.bfloat16),
    (1, 2, 400 - 68, 100, 4, True, 64, 1, 1, 4, torch.bfloat16),
    (1, 2, 20 * 24 - 30, 20, 24, True, 64, 2, 2, 2, torch.bfloat16),
    (1, 2, 20 * 24 - 30, 20, 24, False, 64, 2, 2, 2, torch.float32),
    # later steps through the two-pass L-update and the paired-tile / streaming R-updates
    (1, 2, 140 * 80 - 100, 140, 80, True, 64, 2, 1, 2, torch.bfloat16),
    (1, 1, 200 * 8 - 11, 200, 8, True, 64, 2, 1, 1, torch.bfloat16),
    (1, 1, 52 * 90 - 40, 52, 90, True, 128, 2, 1, 1, torch.bfloat16),
    (1, 1, 30 * 156 - 70, 30, 156, False, 128, 2, 1, 1, torch.bfloat16),
    (1, 2, 6 * 7 - 10, 6, 7, True, 64, 0, 1, 3, torch.float32),
    (1, 2, 6 * 7 - 10, 6, 7, False, 64, 0, 1, 3, torch.bfloat16),
    (1, 1, 5 * 6 - 4, 5, 6, True, 7, 2, 1, 2, torch.bfloat16),
    (1, 1, 5 * 6 - 4, 5, 6, False, 24, 1, 2, 2, torch.float32),
    (1, 2, 1, 8, 8, True, 64, 1, 1, 1, torch.bfloat16),
    (1, 2, 30 * 156 - 200, 30, 156, True, 128, 1, 2, 2, torch.bfloat16),  # position tiles
    (1, 2, 200 * 8 - 20, 200, 8, True, 64, 2, 1, 1, torch.bfloat16),  # two-pass L-update
    (1, 2, 30 * 156 - 100, 30, 156, True, 128, 1, 1, 1, torch.bfloat16),  # streamed groups
]


@pytest.mark.parametrize("B,H,n,b1,b2,front,d,T,c1,c2,dtype", CASES)
def test_padded_parity(cuda_lib, B, H, n, b1, b2, front, d, T, c1, c2, dtype):
    q, k, v = iid_qkv(B, H, n, d, dtype, seed=n + 7 * b2)
    O = cuda_lib.monarch_attn_fwd_padded(q.cuda(), k.cuda(), v.cuda(), b1, b2, T, c1, c2,
                                         pad_front=front)
    cuda_lib.check()
    assert cuda_lib.last_launches() > 0
    ref = monarch_attention(q.double().numpy(), k.double().numpy(), v.double().numpy(), b1, b2,
                            T, c1, c2, n_pad=b1 * b2 - n, pad_front=front)
    Og = O.double().cpu().numpy()
    assert np.isfinite(Og).all()
    err = np.abs(Og - ref).max()
    bound = TOL[dtype] * v.abs().max().item()
    assert err <= bound, f"max err {err:.3e} > {bound:.3e}"


def test_full_grid_is_the_unpadded_forward(cuda_lib):
    q, k, v = (x.cuda() for x in iid_qkv(1, 2, 90 * 52, 128, torch.bfloat16, seed=5))
    a = cuda_lib.monarch_attn_fwd_padded(q, k, v, 90, 52, 1)
    b = cuda_lib.monarch_attn_fwd(q, k, v, 90, 52, 1)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
