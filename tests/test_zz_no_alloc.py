"""The allocation-free entry point against the default one, on the GPU.

monarch_attn_fwd_noalloc serves callers that cannot allocate device memory
when they call (a real-time frame loop, or a host that owns all device memory
through its own pool).  Its scratch is a static device array shared by every
call, so the check runs two calls in a row on one stream and compares each
with monarch_attn_fwd under the parity bar the other GPU tests use
(2e-2 max|V| for bf16).  This file is collected last on purpose.
"""
import pytest
import torch

from structured_sub_quadratic_b200.inputs import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["480p", "vit"])
def test_noalloc_matches_default_entry_on_two_calls(cuda_lib, name):
    wl = WORKLOADS[name]
    q, k, v = (x.cuda() for x in make_inputs(wl))
    ref = cuda_lib.monarch_attn_fwd(q, k, v, wl.b1, wl.b2, wl.T, wl.c1, wl.c2)
    torch.cuda.synchronize()
    bound = 2e-2 * v.float().abs().max().item()
    for _ in range(2):
        out = torch.full_like(q, float("nan"))
        cuda_lib.monarch_attn_fwd_noalloc(q, k, v, wl.b1, wl.b2, wl.T, wl.c1, wl.c2, out=out)
        torch.cuda.synchronize()
        assert torch.isfinite(out).all()
        err = (out.float() - ref.float()).abs().max().item()
        assert err <= bound, f"{err:.3e} > {bound:.3e}"


def test_noalloc_rejects_shapes_beyond_its_scratch(cuda_lib):
    wl = WORKLOADS["720p"]
    q = torch.empty(wl.B, wl.H, wl.N, wl.d, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(cuda_lib.MonarchError) as exc:
        cuda_lib.monarch_attn_fwd_noalloc(q, q, q, wl.b1, wl.b2, wl.T, wl.c1, wl.c2,
                                          out=torch.empty_like(q))
    assert exc.value.status == cuda_lib.MONARCH_ERR_SCRATCH_LIMIT
