"""GPU parity of the tensor-core paths beyond the basic cases.

1. Element-wise comparison with the fp64 oracle at sizes that give every CTA
   of the persistent tensor-core kernel at least three tiles (148 CTAs at
   most: the "next tile loaded during the current tile's last stages" path and
   the split mode's parked z_even are exercised many times per CTA), in every
   mode the kernels have: plain (N = 4096), packed short sequences (N = 256 ..
   2048, 4096 / N of them per 8192-point transform), overlap-save windows
   (partial filters, N >= 32768), the block modes of N = 8192 (two blocks of
   4096, unmasked calls) and N = 16384 (four blocks), the N = 8192 parity
   split (masked calls) and the staged path's row pass.  The launch configuration is the plan's own, as in the benchmark.
2. Closed forms the convolution must reproduce on every tensor-core mode
   (exact results of the definition "FlashFFTConv: Efficient Convolutions for
   Long Sequences with Tensor Cores", summary and "Approach", with the
   dtype-rounded inputs): delta and shifted-delta filters give the (gated,
   shifted) input back; u = 1 gives the running sum of the filter (t + 1 for
   k = 1, a geometric sum for k = r^s); an all-zero block mask gives exactly
   zero and an all-ones mask reproduces the unmasked call bit for bit.
3. The fp16 range guard: inputs at the documented bound stay finite with
   status OK, inputs beyond it set FFTCONV_ERR_RANGE instead of returning
   inf/NaN silently.
"""
import numpy as np
import pytest

import oracle
import workloads as W
from parity_util import assert_close, run_cuda

pytestmark = pytest.mark.gpu

SMS = 148         # CTAs of the persistent tensor-core kernel (B200)


def _inputs(B, H, N, L, dtype, gated, mask_frac=0.0, seed=0, shared_mask=False):
    rng = np.random.default_rng(seed)
    out = {"u": W.round_to(rng.standard_normal((B, H, N), dtype=np.float32), dtype),
           "k": W.round_to(rng.standard_normal((H, L), dtype=np.float32) / np.float32(np.sqrt(L)), dtype),
           "w": None, "v": None, "mask": None}
    if gated:
        out["w"] = W.round_to(rng.standard_normal((B, H, N), dtype=np.float32), dtype)
        out["v"] = W.round_to(rng.standard_normal((B, H, N), dtype=np.float32), dtype)
    if mask_frac > 0:
        out["mask"] = (rng.random((1 if shared_mask else H, N // 32)) >= mask_frac).astype(np.uint8)
    return out


def _compare(inp, dtype, what, order=0, path="tc_fused"):
    y, plan = run_cuda(inp, dtype, order=order)
    assert plan.path_name == path, (what, plan.path_name)
    ref = oracle.fftconv(inp["u"], inp["k"], w=inp["w"], v=inp["v"], mask=inp["mask"])
    e = assert_close(y, ref, dtype, what)
    rms = float(np.sqrt(np.mean(ref ** 2)))
    # the literal max-abs error beside the bound it is held to
    print(f"{what}: rel_l2={e:.2e} max_abs={np.max(np.abs(y - ref)):.3e} (2e-2*rms={2e-2 * rms:.3e})")
    return y


# ------------------------------------------------- many tiles per CTA ---

def test_plain_mode_three_tiles_per_cta():
    B, H, N = 16, 256, 4096
    tiles = H * ((B // 2 + 3) // 4)                     # 4 pairs of one channel per tile
    assert tiles >= 3 * SMS
    _compare(_inputs(B, H, N, N, "bf16", gated=True, seed=1), "bf16", f"plain {tiles} tiles")


def test_plain_mode_ragged_batch_many_tiles():
    # B = 13: six full pairs and an unpaired row per channel, two tiles per
    # channel, the second one ragged
    B, H, N = 13, 240, 4096
    tiles = H * (((B + 1) // 2 + 3) // 4)
    assert tiles >= 3 * SMS
    _compare(_inputs(B, H, N, N, "f16", gated=False, seed=2), "f16", f"plain ragged {tiles} tiles")


@pytest.mark.parametrize("N,B,H,L,gated,dtype", [(1024, 64, 240, 1024, True, "bf16"),
                                                (2048, 16, 480, 2048, False, "f16"),
                                                (512, 27, 450, 300, True, "bf16"),
                                                (256, 33, 450, 256, False, "bf16")])
def test_packed_mode_three_tiles_per_cta(N, B, H, L, gated, dtype):
    pairs_per_tile = 4 * (4096 // N)
    tiles = H * (((B + 1) // 2 + pairs_per_tile - 1) // pairs_per_tile)
    assert tiles >= 3 * SMS
    _compare(_inputs(B, H, N, L, dtype, gated=gated, seed=N + B), dtype, f"packed N={N} B={B} L={L} {tiles} tiles")


def test_packed_mode_rejects_masks():
    import long_sequence_fft_b200 as lsf
    inp = _inputs(2, 2, 1024, 1024, "bf16", gated=False, mask_frac=0.5, seed=9)
    with pytest.raises(lsf.FFTConvError) as ei:
        run_cuda(inp, "bf16", order=0)
    assert ei.value.status == lsf.ERR_UNSUPPORTED


def test_windows_mode_three_tiles_per_cta():
    B, H, N, L = 16, 16, 32768, 2048
    tiles = H * (N // 2048 - 1) * ((B // 2 + 3) // 4)
    assert tiles >= 3 * SMS
    _compare(_inputs(B, H, N, L, "bf16", gated=True, seed=3), "bf16", f"windows {tiles} tiles")


@pytest.mark.parametrize("B,H,L,gated,dtype", [(8, 112, 16384, True, "bf16"),
                                               (7, 128, 9000, False, "f16"),
                                               (8, 112, 4000, True, "bf16")])
def test_four_block_mode_three_tiles_per_cta(B, H, L, gated, dtype):
    """N = 16384: one pair per tile as four blocks of 4096; block b adds the
    earlier blocks' spectra times G_1 .. G_b."""
    N = 16384
    tiles = H * ((B + 1) // 2)
    assert tiles >= 3 * SMS
    _compare(_inputs(B, H, N, L, dtype, gated=gated, seed=L + B + 1), dtype, f"four-block L={L} B={B} {tiles} tiles")


@pytest.mark.parametrize("B,H,L,gated,dtype", [(16, 112, 8192, True, "bf16"),
                                               (13, 128, 5000, False, "f16"),
                                               (16, 112, 2048, True, "bf16"),
                                               (15, 120, 4097, True, "f16")])
def test_two_block_mode_three_tiles_per_cta(B, H, L, gated, dtype):
    """N = 8192 without a mask: two pairs per tile, each as two blocks of 4096
    (block 1 takes block 0's spectrum through shared memory)."""
    N = 8192
    tiles = H * (((B + 1) // 2 + 1) // 2)
    assert tiles >= 3 * SMS
    _compare(_inputs(B, H, N, L, dtype, gated=gated, seed=L + B), dtype, f"two-block L={L} B={B} {tiles} tiles")


@pytest.mark.parametrize("N,B,H,L,dtype", [(1024, 9, 40, 1024, "bf16"),
                                           (4096, 5, 40, 4096, "f16"),
                                           (8192, 7, 24, 3000, "bf16"),
                                           (16384, 3, 16, 16384, "f16")])
def test_output_gate_only(N, B, H, L, dtype):
    """y = v * conv(u, k) with no input gate: calls without w run the
    kernel's ungated build (no gate loads), with or without v."""
    inp = _inputs(B, H, N, L, dtype, gated=True, seed=N + B)
    inp["w"] = None
    _compare(inp, dtype, f"v only N={N} B={B} L={L}")


def test_split_mode_three_tiles_per_cta():
    B, H, N = 16, 128, 8192
    groups = H * ((B // 2 + 3) // 4)
    assert 2 * groups >= 3 * SMS                        # even and odd tile per group
    _compare(_inputs(B, H, N, N, "bf16", gated=True, mask_frac=0.75, seed=4, shared_mask=True), "bf16",
             f"split {2 * groups} tiles")


def test_rows_mode_three_tiles_per_cta():
    B, H, N = 8, 64, 32768
    units = H * (B // 2) * ((2 * N // 8192) // 4)       # rows mode: 4 rows of one pair per tile
    assert units >= 3 * SMS
    _compare(_inputs(B, H, N, N, "f16", gated=True, seed=5), "f16", f"rows {units} tiles", order=0,
             path="tc_staged")


# ------------------------------------------------------- closed forms ---

MODES = [  # (name, N, L, order, path); the split mode runs for masked calls
    ("plain", 4096, 4096, 0, "tc_fused"),
    ("packed1k", 1024, 1024, 0, "tc_fused"),
    ("packed256", 256, 256, 0, "tc_fused"),
    ("windows", 32768, 2048, 0, "tc_fused"),
    ("twoblock", 8192, 8192, 0, "tc_fused"),
    ("fourblock", 16384, 16384, 0, "tc_fused"),
    ("fourblock_partial", 16384, 6000, 0, "tc_fused"),
    ("twoblock_partial", 8192, 3000, 0, "tc_fused"),
    ("split", 8192, 8192, 0, "tc_fused"),
    ("rows", 16384, 16384, 5, "tc_staged"),
]


def _keep_all(name, N):
    """An all-ones block mask (it selects the masked kernel, the parity split,
    at N = 8192 and changes nothing else)."""
    return np.ones((1, N // 32), np.uint8) if name == "split" else None


def _run(u, k, dtype, order, path, w=None, v=None, mask=None):
    inp = {"u": u, "k": k, "w": w, "v": v, "mask": mask}
    y, plan = run_cuda(inp, dtype, order=order)
    assert plan.path_name == path
    return y


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
@pytest.mark.parametrize("name,N,L,order,path", MODES)
def test_delta_filters_return_the_input(name, N, L, order, path, dtype):
    rng = np.random.default_rng(N + L)
    B, H = 3, 2
    u = W.round_to(rng.standard_normal((B, H, N), dtype=np.float32), dtype)
    w = W.round_to(rng.standard_normal((B, H, N), dtype=np.float32), dtype)
    v = W.round_to(rng.standard_normal((B, H, N), dtype=np.float32), dtype)
    x = u.astype(np.float64) * w * v
    k = np.zeros((H, L), np.float32)
    k[:, 0] = 1.0
    m = _keep_all(name, N)
    y = _run(u, k, dtype, order, path, w=w, v=v, mask=m)
    assert_close(y, x, dtype, f"{name}: delta filter")
    # shifted delta (a different shift per channel): y[t] = (u w)[t - d] v[t];
    # at N = 8192 one shift moves block 0 entirely into block 1 and the other
    # gives block 1 outputs from both blocks' inputs (both two-block terms)
    d = {8192: [min(L - 1, 4095), 2000], 16384: [min(L - 1, 12289), 5000]}.get(N, [min(5, L - 1), min(L - 1, 1500)])
    k = np.zeros((H, L), np.float32)
    ref = np.zeros((B, H, N))
    for h in range(H):
        k[h, d[h]] = 1.0
        ref[:, h, d[h]:] = (u[:, h, :N - d[h]].astype(np.float64) * w[:, h, :N - d[h]]) * v[:, h, d[h]:]
    y = _run(u, k, dtype, order, path, w=w, v=v, mask=m)
    assert_close(y, ref, dtype, f"{name}: shifted delta")


@pytest.mark.parametrize("name,N,L,order,path", MODES)
def test_running_sums_of_the_filter(name, N, L, order, path):
    """u = 1: y[t] = sum_{s <= min(t, L-1)} k[s]; k = 1 gives t + 1 (capped at
    L for a partial filter) and k = r^s the geometric sum."""
    dtype = "f16" if N > 4096 else "bf16"
    B, H = 2, 2
    u = np.ones((B, H, N), np.float32)
    t = np.arange(N)
    m = _keep_all(name, N)
    k1 = np.ones((H, L), np.float32)
    y = _run(u, k1, dtype, order, path, mask=m)
    ref = np.broadcast_to(np.minimum(t, L - 1) + 1.0, (B, H, N))
    assert_close(y, ref, dtype, f"{name}: u = k = 1")
    r = np.array([0.999, 0.99], np.float64)
    kg = W.round_to((r[:, None] ** np.arange(L)[None, :]).astype(np.float32), dtype)
    y = _run(u, kg, dtype, order, path, mask=m)
    cs = np.cumsum(kg.astype(np.float64), axis=1)        # the rounded taps' running sums
    ref = np.broadcast_to(cs[:, np.minimum(t, L - 1)][None], (B, H, N))
    assert_close(y, ref, dtype, f"{name}: geometric filter")
    # and the geometric closed form itself, within the rounding of the taps
    closed = (1 - r[:, None] ** (np.minimum(t, L - 1)[None, :] + 1)) / (1 - r[:, None])
    assert np.max(np.abs(cs[:, np.minimum(t, L - 1)] - closed) / closed) < 5e-3


@pytest.mark.parametrize("name,N,order,path", [("split", 8192, 0, "tc_fused"), ("rows", 16384, 5, "tc_staged")])
def test_zero_and_full_masks_on_tensor_cores(name, N, order, path):
    inp = _inputs(3, 2, N, N, "bf16", gated=True, seed=N)
    inp["mask"] = np.zeros((1, N // 32), np.uint8)
    y, plan = run_cuda(inp, "bf16", order=order)
    assert plan.path_name == path
    assert np.max(np.abs(y)) == 0.0, f"{name}: all-zero mask must give exact zeros"
    inp["mask"] = np.full((2, N // 32), 9, np.uint8)     # any nonzero byte keeps the block
    y1, _ = run_cuda(inp, "bf16", order=order)
    if name == "split":
        # at N = 8192 an unmasked call runs the two-block kernel instead: the
        # all-ones mask equals another all-ones mask bit for bit, and the
        # oracle's unmasked result within the tolerance
        inp["mask"] = np.ones((1, N // 32), np.uint8)
        y2, _ = run_cuda(inp, "bf16", order=order)
        assert np.array_equal(y1, y2), f"{name}: all-ones masks must agree bit for bit"
        assert_close(y1, oracle.fftconv(inp["u"], inp["k"], w=inp["w"], v=inp["v"]), "bf16", f"{name}: all-ones")
        return
    inp["mask"] = None
    y2, _ = run_cuda(inp, "bf16", order=order)
    assert np.array_equal(y1, y2), f"{name}: all-ones mask must equal the unmasked call"


# --------------------------------------------------------- fp16 range ---

def _status_after(u, k, dtype, order, N, L, mask=None):
    import long_sequence_fft_b200 as lsf
    import torch
    from parity_util import to_dev
    plan = lsf.Plan(N, u.shape[1], dtype, order=order, L=L)
    Kf = plan.precompute(to_dev(k, dtype))
    y = plan.forward(to_dev(u, dtype), Kf, mask=None if mask is None else torch.from_numpy(mask).cuda())
    torch.cuda.synchronize()
    status = lsf.library().fftconv_device_status(plan.handle, None)
    again = lsf.library().fftconv_device_status(plan.handle, None)
    return y.float().cpu().numpy().astype(np.float64), status, again, plan


@pytest.mark.parametrize("name,N,L,order,path,edge,beyond", [
    ("plain", 4096, 4096, 0, "tc_fused", 90.0, 1500.0),
    ("packed1k", 1024, 1024, 0, "tc_fused", 90.0, 6000.0),     # B = 2: one segment of 1024 per row
    ("windows", 32768, 2048, 0, "tc_fused", 90.0, 1500.0),
    ("fourblock", 16384, 16384, 0, "tc_fused", 90.0, 1500.0),
    ("twoblock", 8192, 8192, 0, "tc_fused", 90.0, 1500.0),
    ("split", 8192, 8192, 0, "tc_fused", 90.0, 3000.0),
    ("rows", 16384, 16384, 5, "tc_staged", 90.0, 2000.0),
])
def test_fp16_range_guard(name, N, L, order, path, edge, beyond):
    import long_sequence_fft_b200 as lsf
    B, H = 2, 1
    k = np.zeros((H, L), np.float32)
    k[:, 0] = 1.0                                        # delta: y = u, flat spectrum
    # at the documented data-independent bound: finite, status OK, exact result
    u = np.full((B, H, N), edge, np.float32)
    m = _keep_all(name, N)
    y, status, again, plan = _status_after(u, k, "bf16", order, N, L, m)
    assert plan.path_name == path
    assert status == lsf.OK and np.isfinite(y).all()
    assert_close(y, u.astype(np.float64), "bf16", f"{name}: constant {edge} at the bound")
    # a constant input far beyond it overflows the fp16 forward transform: the
    # call reports FFTCONV_ERR_RANGE (and the status word resets on read)
    u = np.full((B, H, N), beyond, np.float32)
    y, status, again, _ = _status_after(u, k, "bf16", order, N, L, m)
    assert status == lsf.ERR_RANGE, (name, status)
    assert again == lsf.OK
    assert not np.isfinite(y).all()


@pytest.mark.parametrize("name,N,T,amp", [("plain", 4096, 4093, 2.0e4),
                                          ("packed1k", 1024, 1021, 4.0e4),
                                          ("twoblock", 8192, 4093, 2.0e4)])
def test_fp16_range_guard_inverse_stage(name, N, T, amp):
    """An overflow that only an inverse stage meets, confined to one residue.

    The fused kernel's 8192-point transform indexes time as t = 256 j1 + 8 l +
    j3.  A linear chirp u of T samples and its matched filter k (u reversed,
    amplitude 1) compress into one sample at t = T - 1, whose (l, j3) is
    (31, 4) for both lengths here.  Per unit amplitude the largest forward
    fp16 value is 2.45 (T = 4093) or 0.67 (T = 1021), the S2' output at that
    (l, j3) 5.93 or 2.97, every other S2' value below 0.12: at `amp` the
    forward stages stay below 49k and that one S2' value passes 65504.  Only
    the outputs of that (l, j3) become non-finite (16 of the 4096 of a block,
    none with j3 = 0), and the call must report FFTCONV_ERR_RANGE.  At a
    quarter of `amp` nothing overflows and the result is the oracle's."""
    import long_sequence_fft_b200 as lsf
    B, H = 2, 1
    t = np.arange(T)
    chirp = np.cos(np.pi * t.astype(np.float64) ** 2 / (2 * T))
    k = np.zeros((H, T), np.float32)
    k[0] = chirp[::-1]
    u = np.zeros((B, H, N), np.float32)
    for scale, overflow in ((0.25, False), (1.0, True)):
        u[0, 0, :T] = amp * scale * chirp
        ub = W.round_to(u, "bf16")
        kb = W.round_to(k, "bf16")
        y, status, again, plan = _status_after(ub, kb, "bf16", 0, N, T)
        assert plan.path_name == "tc_fused"
        if not overflow:
            assert status == lsf.OK and np.isfinite(y).all(), (name, status)
            assert_close(y, oracle.fftconv(ub, kb), "bf16", f"{name}: matched chirp below the overflow")
            continue
        assert status == lsf.ERR_RANGE, (name, status)
        assert again == lsf.OK
        bad = np.nonzero(~np.isfinite(y))[-1]
        assert bad.size > 0, name
        assert np.all(bad % 256 == 8 * 31 + 4), (name, sorted(set((bad % 256).tolist())))


# ------------------------------------------------ block-mode edge cases ---

@pytest.mark.parametrize("N,B,H,L,dtype", [(8192, 1, 1, 8192, "bf16"),      # one unpaired row
                                           (8192, 3, 1, 1, "f16"),          # L = 1, a ragged pair
                                           (16384, 1, 2, 16384, "f16"),
                                           (16384, 2, 1, 1, "bf16"),
                                           (16384, 5, 3, 4097, "bf16")])    # G_2 = G_3 = 0 skipped
def test_block_modes_small_and_ragged(N, B, H, L, dtype):
    _compare(_inputs(B, H, N, L, dtype, gated=(B % 2 == 1), seed=N + B + L), dtype, f"blocks N={N} B={B} L={L}")


def test_block_modes_empty_batch():
    import torch
    import long_sequence_fft_b200 as lsf
    for N in (8192, 16384):
        plan = lsf.Plan(N, 2, "bf16")
        Kf = plan.precompute(torch.zeros((2, N), dtype=torch.bfloat16, device="cuda"))
        u = torch.zeros((0, 2, N), dtype=torch.bfloat16, device="cuda")
        y = plan.forward(u, Kf)
        torch.cuda.synchronize()
        assert y.shape == (0, 2, N) and plan.device_status() == 0
