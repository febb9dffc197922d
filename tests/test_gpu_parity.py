"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle,
element by element, on the same seeded inputs.

Bar: max|O_gpu - O_oracle| <= 1e-4 max|V| for fp32 inputs and
<= 2e-2 max|V| for bf16 inputs.  The oracle reads the exact values the GPU
receives (bf16 inputs are widened to float64).
"""
import numpy as np
import pytest
import torch

from oracle import monarch_attention
from structured_sub_quadratic_b200.inputs import WORKLOADS, iid_qkv, make_inputs, video_qkv

pytestmark = pytest.mark.gpu

TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}


def gpu_forward(api, q, k, v, b1, b2, T, c1=1, c2=1):
    qd, kd, vd = (x.cuda() for x in (q, k, v))
    out = api.monarch_attn_fwd(qd, kd, vd, b1, b2, T, c1, c2)
    api.check()
    assert api.last_launches() > 0
    return out.double().cpu().numpy()


def oracle_forward(q, k, v, b1, b2, T, c1=1, c2=1):
    return monarch_attention(q.double().numpy(), k.double().numpy(), v.double().numpy(),
                             b1, b2, T, c1, c2)


def assert_parity(O, ref, v, dtype):
    bound = TOL[dtype] * v.abs().max().item()
    err = np.abs(O - ref).max()
    assert np.isfinite(O).all()
    assert err <= bound, f"max err {err:.3e} > {bound:.3e}"
    return err


@pytest.mark.parametrize("name", ["tiny", "vit", "sweep256", "sweep1k", "sweep4k", "sweep16k",
                                  "480p"])
def test_config_parity(cuda_lib, name):
    wl = WORKLOADS[name]
    q, k, v = make_inputs(wl)
    O = gpu_forward(cuda_lib, q, k, v, wl.b1, wl.b2, wl.T, wl.c1, wl.c2)
    ref = oracle_forward(q, k, v, wl.b1, wl.b2, wl.T, wl.c1, wl.c2)
    assert_parity(O, ref, v, wl.dtype)


def test_720p_tiled_parity_on_two_heads(cuda_lib):
    wl = WORKLOADS["720p"]
    q, k, v = make_inputs(wl)
    O = gpu_forward(cuda_lib, q, k, v, wl.b1, wl.b2, wl.T, wl.c1, wl.c2)
    for h in (0, wl.H - 1):
        sl = slice(h, h + 1)
        ref = oracle_forward(q[:, sl], k[:, sl], v[:, sl], wl.b1, wl.b2, wl.T, wl.c1, wl.c2)
        assert_parity(O[:, sl], ref, v[:, sl], wl.dtype)


EDGE = [
    # B, H, b1, b2, d, T, c1, c2
    (1, 2, 1, 24, 64, 1, 1, 1),      # one chunk: exact attention
    (1, 2, 24, 1, 64, 2, 1, 1),      # one position per chunk
    (2, 3, 7, 9, 64, 2, 3, 2),       # uneven groups, two steps
    (1, 2, 9, 7, 128, 3, 9, 7),      # every sub-tile 1 x 1
    (1, 1, 5, 6, 24, 1, 2, 2),       # d not a multiple of 32
    (1, 1, 5, 6, 7, 2, 1, 2),        # d odd: unaligned rows, scalar loads
    (1, 2, 6, 6, 256, 1, 1, 1),      # largest d
    (3, 1, 33, 35, 64, 1, 1, 1),     # ragged against 32-wide chunks
    (1, 1, 100, 3, 32, 2, 2, 1),     # long L rows
    (1, 2, 7, 7, 64, 0, 1, 3),       # T = 0 with uneven column groups
    (1, 1, 4, 70, 64, 1, 1, 3),      # long R rows in groups
    (1, 2, 200, 8, 64, 1, 1, 1),     # more than 128 keys per L row: multi-tile output kernel
    (1, 1, 70, 20, 128, 2, 2, 2),    # 140 keys per L row in row groups, two steps
    (1, 1, 45, 64, 128, 1, 1, 1),    # paired R tiles with 64 positions, odd sub-item count
    (2, 3, 5, 7, 64, 2, 1, 1),       # small head kept in shared memory, two steps
    (1, 2, 16, 13, 64, 3, 1, 1),     # largest small-head blocks, three steps
    (1, 1, 1, 9, 64, 2, 1, 1),       # small head, one row block
    (1, 1, 12, 1, 64, 2, 1, 1),      # small head, one position
    (1, 2, 30, 156, 128, 1, 2, 2),   # b2 > 128: two position tiles, 78-key groups
    (1, 2, 12, 200, 64, 1, 1, 4),    # two position tiles, 50-key groups
    (1, 1, 6, 300, 64, 2, 2, 3),     # three position tiles, 100-key groups, two steps
    (1, 2, 30, 156, 128, 1, 1, 1),   # 156-key groups: streamed in 128-key sub-tiles
    (1, 1, 8, 300, 64, 1, 1, 1),     # 300-key groups, three sub-tiles, three position tiles
    (1, 1, 6, 130, 128, 2, 1, 1),    # 130-key groups, two steps
    (1, 2, 10, 200, 64, 1, 2, 1),    # 200-key groups in two row groups
    (1, 1, 3, 1560, 128, 1, 1, 1),   # the (f,hw) blocks of the 480p latent: 13 position tiles
    # unpaired R tiles (64 < b2 <= 128) with d = 128
    (1, 2, 33, 128, 128, 1, 1, 2),   # 128 positions, 64-key groups
    (1, 1, 21, 100, 128, 1, 2, 2),   # 50-key groups in a 64-key tile, uneven row groups
    (2, 1, 17, 96, 128, 2, 1, 3),    # 32-key groups, two steps (Kt-only first R-update)
    (1, 1, 9, 80, 128, 1, 1, 5),     # 16-key groups
    (1, 1, 400, 72, 128, 1, 1, 2),   # 800 sub-items over the SMs: several tiles per warpgroup
    # unpaired R tiles of 65-96 keys (two K|V slots at d = 128)
    (1, 2, 20, 90, 64, 2, 1, 1),     # 90-key groups in 96-key tiles, two steps
    (1, 1, 16, 75, 128, 1, 1, 1),    # 75-key groups in 80-key tiles
    (2, 1, 24, 96, 128, 2, 1, 1),    # 96-key groups, full tiles, two steps
]


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("B,H,b1,b2,d,T,c1,c2", EDGE)
def test_edge_shapes(cuda_lib, dtype, B, H, b1, b2, d, T, c1, c2):
    q, k, v = iid_qkv(B, H, b1 * b2, d, dtype, seed=b1 * 100 + b2)
    O = gpu_forward(cuda_lib, q, k, v, b1, b2, T, c1, c2)
    ref = oracle_forward(q, k, v, b1, b2, T, c1, c2)
    assert_parity(O, ref, v, dtype)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_separable_video_logits_are_near_exact(cuda_lib, dtype):
    """Pure separable logits with aligned blocks: the method is exact at T=1,
    so the GPU output must match dense attention within the same bar."""
    latent = (3, 10, 16)
    q, k, v = video_qkv(1, 2, latent, 64, dtype, seed=7, noise=False)
    O = gpu_forward(cuda_lib, q, k, v, 30, 16, 1)
    qd, kd, vd = (x.double() for x in (q, k, v))
    E = torch.softmax(qd @ kd.transpose(-1, -2) / 8.0, dim=-1) @ vd
    assert_parity(O, E.numpy(), v, dtype)


def test_host_buffer_entry_matches_device_entry(cuda_lib):
    wl = WORKLOADS["sweep1k"]
    q, k, v = make_inputs(wl)
    qh, kh, vh = (x.pin_memory() for x in (q, k, v))
    out = torch.empty_like(qh).pin_memory()
    cuda_lib.monarch_attn_fwd_host(qh, kh, vh, out, wl.b1, wl.b2, wl.T)
    O = gpu_forward(cuda_lib, q, k, v, wl.b1, wl.b2, wl.T)
    np.testing.assert_array_equal(out.double().numpy(), O)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_host_buffer_entry_pipelines_head_groups(cuda_lib, dtype):
    """The host-buffer entry copies and computes in groups of heads (at least
    32 MiB of input each) on three streams: with 26 heads of 16 K tokens (9
    groups of up to 3 heads in fp32, 4 of up to 7 in bf16) and two different
    input sets back to back, each result equals the device entry's bit for
    bit."""
    B, H, b1, b2, d, T = 2, 13, 128, 128, 64, 1
    for seed in (21, 22):
        q, k, v = iid_qkv(B, H, b1 * b2, d, dtype, seed=seed)
        qh, kh, vh = (x.pin_memory() for x in (q, k, v))
        out = torch.empty_like(qh).pin_memory()
        cuda_lib.monarch_attn_fwd_host(qh, kh, vh, out, b1, b2, T)
        O = gpu_forward(cuda_lib, q, k, v, b1, b2, T)
        np.testing.assert_array_equal(out.double().numpy(), O)


def test_repeat_calls_are_deterministic(cuda_lib):
    wl = WORKLOADS["480p"]
    q, k, v = (x.cuda() for x in make_inputs(wl))
    a = cuda_lib.monarch_attn_fwd(q, k, v, wl.b1, wl.b2, wl.T)
    b = cuda_lib.monarch_attn_fwd(q, k, v, wl.b1, wl.b2, wl.T)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_tensor_core_and_simt_kernels_agree(cuda_lib):
    """The bf16 entry (tensor-core kernels) against the fp32 entry (SIMT
    kernels) on the same values: they differ only by the bf16 rounding of
    the intermediates, within the bf16 bar."""
    wl = WORKLOADS["480p"]
    q, k, v = make_inputs(wl)
    O_tc = gpu_forward(cuda_lib, q, k, v, wl.b1, wl.b2, wl.T)
    O_simt = gpu_forward(cuda_lib, q.float(), k.float(), v.float(), wl.b1, wl.b2, wl.T)
    assert_parity(O_tc, O_simt, v, wl.dtype)


def test_bounded_wait_timeout_is_reported_and_context_survives(cuda_lib):
    """A device wait that nothing satisfies gives up after its limit, sets the
    status word and returns; the host reads MONARCH_ERR_DEVICE_TIMEOUT once,
    and the context keeps running forward passes."""
    cuda_lib.check()  # clean slate
    cuda_lib.selftest_timeout(20_000_000)  # 20 ms
    with pytest.raises(cuda_lib.MonarchError) as exc:
        cuda_lib.check()
    assert exc.value.status == cuda_lib.MONARCH_ERR_DEVICE_TIMEOUT
    cuda_lib.check()  # the flag was cleared by the read
    q, k, v = iid_qkv(1, 2, 64, 64, torch.bfloat16, seed=9)
    O = gpu_forward(cuda_lib, q, k, v, 8, 8, 1)
    assert_parity(O, oracle_forward(q, k, v, 8, 8, 1), v, torch.bfloat16)


def test_back_to_back_calls_consume_previous_output(cuda_lib):
    """Stream ordering across calls: the next call's queries (then keys) are
    the previous call's output, issued without a host synchronisation, so an
    early start of any kernel of the second call would read stale rows."""
    wl = WORKLOADS["480p"]
    q, k, v = make_inputs(wl)
    qd, kd, vd = (x.cuda() for x in (q, k, v))
    o1 = cuda_lib.monarch_attn_fwd(qd, kd, vd, wl.b1, wl.b2, wl.T)
    o2 = cuda_lib.monarch_attn_fwd(o1, kd, vd, wl.b1, wl.b2, wl.T)
    o3 = cuda_lib.monarch_attn_fwd(qd, o2, vd, wl.b1, wl.b2, wl.T)
    cuda_lib.check()
    o1c, o2c = o1.cpu(), o2.cpu()
    assert_parity(o2.double().cpu().numpy(), oracle_forward(o1c, k, v, wl.b1, wl.b2, wl.T), v,
                  wl.dtype)
    assert_parity(o3.double().cpu().numpy(), oracle_forward(q, o2c, v, wl.b1, wl.b2, wl.T), v,
                  wl.dtype)


# Aligned video layouts: Monarch token m is raster token perm[m], with the
# latent's (f, h, w) axes taken in the layout's order.
LAYOUT_AXES = {"fh,w": (0, 1, 2), "w,fh": (2, 0, 1), "f,hw": (0, 1, 2), "hw,f": (1, 2, 0),
               "fw,h": (0, 2, 1), "h,fw": (1, 0, 2)}


def layout_oracle(q, k, v, latent, layout, T, c1=1, c2=1):
    f, h, w = latent
    perm = np.arange(f * h * w).reshape(f, h, w).transpose(LAYOUT_AXES[layout]).reshape(-1)
    sizes = [latent[a] for a in LAYOUT_AXES[layout]]
    split = 2 if layout in ("fh,w", "hw,f", "fw,h") else 1
    b1 = int(np.prod(sizes[:split]))
    ref_m = oracle_forward(q[..., perm, :], k[..., perm, :], v[..., perm, :], b1,
                           f * h * w // b1, T, c1, c2)
    ref = np.empty_like(ref_m)
    ref[..., perm, :] = ref_m
    return ref


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("layout", list(LAYOUT_AXES))
def test_video_layouts_match_the_permuted_oracle(cuda_lib, dtype, layout):
    latent = (2, 6, 8)
    q, k, v = video_qkv(1, 2, latent, 64, dtype, seed=11)
    O = cuda_lib.monarch_attn_fwd_video(q.cuda(), k.cuda(), v.cuda(), *latent, layout, 1)
    cuda_lib.check()
    assert_parity(O.double().cpu().numpy(), layout_oracle(q, k, v, latent, layout, 1), v, dtype)


@pytest.mark.parametrize("layout,T,c", [("w,fh", 1, 1), ("hw,f", 1, 1), ("h,fw", 2, 2)])
def test_video_layouts_on_the_480p_latent(cuda_lib, layout, T, c):
    """The 480p latent (3, 30, 52), two heads, bf16: (w,fh) is 52 x 90 blocks
    (wide column groups), (hw,f) 1560 x 3 (long L rows), (h,fw) tiled."""
    latent = (3, 30, 52)
    q, k, v = video_qkv(1, 2, latent, 128, torch.bfloat16, seed=12)
    O = cuda_lib.monarch_attn_fwd_video(q.cuda(), k.cuda(), v.cuda(), *latent, layout, T, c, c)
    cuda_lib.check()
    assert_parity(O.double().cpu().numpy(), layout_oracle(q, k, v, latent, layout, T, c, c), v,
                  torch.bfloat16)


def test_injected_allocation_failure_is_reported_and_recovers(cuda_lib, monkeypatch):
    """Host-side fault injection: with MONARCH_ATTN_FAIL_ALLOC=1 the workspace
    allocation of a call fails with MONARCH_ERR_NO_MEMORY (no device call);
    without it the next call allocates and runs."""
    q, k, v = iid_qkv(1, 2, 64, 64, torch.bfloat16, seed=13)
    qd, kd, vd = (x.cuda() for x in (q, k, v))
    torch.cuda.synchronize()
    cuda_lib.release_workspace()
    monkeypatch.setenv("MONARCH_ATTN_FAIL_ALLOC", "1")
    with pytest.raises(cuda_lib.MonarchError) as exc:
        cuda_lib.monarch_attn_fwd(qd, kd, vd, 8, 8, 1)
    assert exc.value.status == cuda_lib.MONARCH_ERR_NO_MEMORY
    monkeypatch.delenv("MONARCH_ATTN_FAIL_ALLOC")
    O = gpu_forward(cuda_lib, q, k, v, 8, 8, 1)
    assert_parity(O, oracle_forward(q, k, v, 8, 8, 1), v, torch.bfloat16)


# Later steps (T >= 2) on the tensor cores: the non-final L-update with the
# aggregation L^T Q, then R-updates from per-sub-item queries.  Each case must
# match the oracle and must not launch any SIMT kernel.
LATER_STEPS = [
    # B, H, b1, b2, d, T, c1, c2, inputs
    (1, 2, 90, 52, 128, 2, 1, 1, "video"),   # the 480p latent (3, 30, 52), paired R tiles
    (1, 2, 90, 52, 128, 3, 1, 1, "video"),
    (1, 3, 64, 64, 64, 2, 1, 1, "iid"),      # sweep 4K shape
    (1, 2, 60, 80, 128, 2, 1, 2, "iid"),     # unpaired R tiles (80 positions, 40-key groups)
    (2, 2, 40, 48, 64, 3, 2, 2, "iid"),      # tiled, three steps
    (1, 2, 45, 20, 128, 2, 3, 2, "iid"),     # tiled with 15-row groups
    # two-pass L-update: rows of more than 128 keys or groups of more than 128 rows
    (1, 2, 70, 20, 128, 2, 2, 2, "iid"),     # 140 keys per row
    (1, 1, 200, 8, 64, 2, 1, 1, "iid"),      # 200 keys, 200-row groups (two row tiles)
    (1, 1, 260, 40, 128, 3, 2, 2, "iid"),    # 520 keys, 130-row groups, paired R tiles
    (1, 1, 140, 80, 64, 2, 1, 2, "iid"),     # 280 keys, unpaired R tiles
    # R-update of the later steps in the paired-tile (<= 96 keys) and streaming kernels
    (1, 2, 64, 128, 64, 2, 1, 1, "iid"),     # 128-key groups (the 16K sweep's shape, 64 chunks)
    (1, 2, 52, 90, 128, 2, 1, 1, "iid"),     # 90-key groups (the (w,fh) blocks of the 480p latent)
    (1, 1, 30, 156, 128, 3, 2, 2, "iid"),    # 78-key groups over two position tiles, three steps
    (1, 1, 30, 156, 128, 2, 1, 1, "iid"),    # 156-key groups, streamed in 128-key sub-tiles
    (1, 1, 6, 300, 64, 2, 1, 2, "iid"),      # 150-key groups, three position tiles
]


@pytest.mark.parametrize("B,H,b1,b2,d,T,c1,c2,kind", LATER_STEPS)
def test_later_steps_on_tensor_cores(cuda_lib, B, H, b1, b2, d, T, c1, c2, kind):
    if kind == "video":
        q, k, v = video_qkv(B, H, (3, 30, 52), d, torch.bfloat16, seed=3)
    else:
        q, k, v = iid_qkv(B, H, b1 * b2, d, torch.bfloat16, seed=b1 + b2 + T)
    cuda_lib.timing_read()
    cuda_lib.timing_enable(True)
    try:
        O = gpu_forward(cuda_lib, q, k, v, b1, b2, T, c1, c2)
        names = set(cuda_lib.timing_read())
    finally:
        cuda_lib.timing_enable(False)
    assert "tc_l_update" in names and not any(n.startswith("simt") for n in names), names
    if b1 * c2 > 128 or -(-b1 // c1) > 128:
        assert "tc_l_stats" in names, names
    assert_parity(O, oracle_forward(q, k, v, b1, b2, T, c1, c2), v, torch.bfloat16)


def test_more_than_128_positions_run_on_tensor_cores(cuda_lib):
    """The (h,fw) layout of the 480p latent in 2 x 2 tiles: b2 = 156 positions
    in two 128-row tiles of the R-update, no SIMT kernel."""
    q, k, v = video_qkv(1, 2, (3, 30, 52), 128, torch.bfloat16, seed=12)
    cuda_lib.timing_read()
    cuda_lib.timing_enable(True)
    try:
        O = gpu_forward(cuda_lib, q, k, v, 30, 156, 1, 2, 2)
        names = set(cuda_lib.timing_read())
    finally:
        cuda_lib.timing_enable(False)
    assert "tc_r_update" in names and not any(n.startswith("simt") for n in names), names
    assert_parity(O, oracle_forward(q, k, v, 30, 156, 1, 2, 2), v, torch.bfloat16)


def test_streamed_groups_rescale_when_the_max_grows(cuda_lib):
    """Column groups of 300 keys whose last 128-key sub-tile holds much larger
    logits, so that it raises the running max by more than 2^8 in most rows
    and the accumulated [Kt | Y] rows are rescaled."""
    b1, b2, d = 6, 300, 64
    q, k, v = iid_qkv(1, 2, b1 * b2, d, torch.float32, seed=31)
    scale = torch.where(torch.arange(b2) >= 256, 6.0, 1.0)  # the last sub-tile dominates
    k = (k.view(1, 2, b1, b2, d) * scale.view(1, 1, 1, b2, 1)).view(1, 2, b1 * b2, d)
    q, k, v = (x.to(torch.bfloat16) for x in (q, k, v))
    O = gpu_forward(cuda_lib, q, k, v, b1, b2, 1)
    assert_parity(O, oracle_forward(q, k, v, b1, b2, 1), v, torch.bfloat16)


@pytest.mark.parametrize("layout,latent,T,c", [("w,fh", (2, 6, 8), 1, 1), ("w,fh", (2, 6, 8), 2, 2),
                                               ("hw,f", (2, 6, 8), 2, 1),
                                               ("w,fh", (3, 30, 52), 1, 1),
                                               ("hw,f", (3, 30, 52), 1, 1)])
def test_transposed_layouts_run_in_place(cuda_lib, layout, latent, T, c):
    """(w,fh) and (hw,f) are the transpose of Monarch order: the tensor-core
    kernels read q, k, v and write out in raster order, with no permute
    launch, and match the oracle on the permuted tokens."""
    d = 64 if latent[0] == 2 else 128
    q, k, v = video_qkv(1, 2, latent, d, torch.bfloat16, seed=13)
    cuda_lib.timing_read()
    cuda_lib.timing_enable(True)
    try:
        O = cuda_lib.monarch_attn_fwd_video(q.cuda(), k.cuda(), v.cuda(), *latent, layout, T, c, c)
        cuda_lib.check()
        names = set(cuda_lib.timing_read())
    finally:
        cuda_lib.timing_enable(False)
    assert "permute_rows" not in names and not any(n.startswith("simt") for n in names), names
    assert_parity(O.double().cpu().numpy(), layout_oracle(q, k, v, latent, layout, T, c, c), v,
                  torch.bfloat16)


# Groups too small for the tensor-core tiles run on the CUDA cores (one warp
# per group): the step-one aggregation for row groups of <= 16 rows, the
# R-update for column groups of <= 8 keys over <= 32 positions, the output
# for rows of <= 8 keys.  Each case names the cc_* kernels it must launch.
SMALL_GROUPS = [
    # B, H, b1, b2, d, T, c1, c2, expected CUDA-core kernels
    (1, 2, 60, 3, 128, 1, 1, 1, {"cc_r_update"}),                # (hw,f)-like: 3-key groups
    (1, 2, 3, 40, 128, 1, 1, 1, {"cc_init_qt", "cc_l_output"}),  # (f,hw)-like: 3-key rows
    (2, 1, 4, 6, 64, 1, 2, 2, {"cc_init_qt", "cc_r_update", "cc_l_output"}),  # tiled, 8-key rows
    (1, 2, 5, 4, 128, 2, 1, 1, {"cc_init_qt", "cc_r_update", "cc_l_output"}),  # two steps
    (1, 1, 20, 32, 64, 3, 2, 4, {"cc_init_qt", "cc_r_update"}),  # 8-key groups, 32 positions
    (1, 1, 7, 5, 128, 1, 7, 1, {"cc_init_qt", "cc_r_update", "cc_l_output"}),  # 1-row groups
    (1, 2, 600, 3, 128, 1, 1, 1, {"cc_init_qt", "cc_r_update"}),  # 6 long row groups: clusters
    (2, 1, 520, 4, 64, 2, 2, 1, {"cc_init_qt", "cc_r_update"}),   # the same, d = 64, tiled, T = 2
]


@pytest.mark.parametrize("B,H,b1,b2,d,T,c1,c2,cc", SMALL_GROUPS)
def test_small_groups_run_on_cuda_cores(cuda_lib, B, H, b1, b2, d, T, c1, c2, cc):
    q, k, v = iid_qkv(B, H, b1 * b2, d, torch.bfloat16, seed=7 * b1 + b2 + T)
    cuda_lib.timing_read()
    cuda_lib.timing_enable(True)
    try:
        O = gpu_forward(cuda_lib, q, k, v, b1, b2, T, c1, c2)
        names = set(cuda_lib.timing_read())
    finally:
        cuda_lib.timing_enable(False)
    assert {n for n in names if n.startswith("cc_")} == cc, names
    assert not any(n.startswith("simt") for n in names), names
    assert_parity(O, oracle_forward(q, k, v, b1, b2, T, c1, c2), v, torch.bfloat16)
