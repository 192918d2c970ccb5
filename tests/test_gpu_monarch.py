"""GPU parity of the Monarch-aligned frequency-sparse forward
(fftconv_forward_monarch) against the oracle's per-bin masked route.

"FlashFFTConv: Efficient Convolutions for Long Sequences with Tensor Cores",
"Approach": frequency-sparse convolutions skip blocks of the Monarch matrix
products; "Key results": up to 79% frequency sparsity.  For N = 4096 the
kernel's 8192-point spectrum index is f = c1 + 32 c2 + 1024 c3; a keep set
over the middle digit c2 selects the bins (a bin is used when its c2 and its
mirror's c2 are kept: workloads.monarch_binmask), and the kernel skips the
tensor-core products and epilogue work of the masked c2."""
import numpy as np
import pytest

import oracle
import workloads as W
from parity_util import assert_close, to_dev

pytestmark = pytest.mark.gpu

SMS = 148


def _inputs(B, H, N, dtype, gated, seed):
    rng = np.random.default_rng(seed)
    r = lambda shape: W.round_to(rng.standard_normal(shape, dtype=np.float32), dtype)
    u = r((B, H, N))
    k = W.round_to(rng.standard_normal((H, N), dtype=np.float32) / np.float32(np.sqrt(N)), dtype)
    return u, k, (r((B, H, N)) if gated else None), (r((B, H, N)) if gated else None)


def _run(u, k, w, v, keep, dtype):
    import torch
    import long_sequence_fft_b200 as lsf
    B, H, N = u.shape
    plan = lsf.Plan(N, H, dtype)
    assert plan.path_name == "tc_fused"
    Kf = plan.precompute(to_dev(k, dtype))
    y = plan.forward_monarch(to_dev(u, dtype), Kf, keep, w=to_dev(w, dtype), v=to_dev(v, dtype))
    torch.cuda.synchronize()
    assert plan.device_status() == 0
    return y.float().cpu().numpy().astype(np.float64), plan, Kf


KEEPS = [0xF000000F,      # c2 in {0..3, 28..31}: 75% sparse, closed under c2 -> 31 - c2
         0x80000001,      # c2 in {0, 31}: 94% sparse
         0x0000FFFF,      # c2 < 16: not closed, the mirror rule masks more
         0x00FF00FF,      # two whole K steps of the 32-point stage
         0x12345678]      # scattered


@pytest.mark.parametrize("keep", KEEPS)
@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_monarch_mask_matches_oracle_bins(keep, dtype):
    B, H, N = 3, 2, 4096
    u, k, w, v = _inputs(B, H, N, dtype, gated=True, seed=keep & 0xFFFF)
    y, _, _ = _run(u, k, w, v, keep, dtype)
    ref = oracle.fftconv_bins(u, k, W.monarch_binmask(keep, N), w=w, v=v)
    assert_close(y, ref, dtype, f"monarch keep=0x{keep:08X} {dtype}")


def test_monarch_three_tiles_per_cta():
    B, H, N = 16, 256, 4096
    tiles = H * ((B // 2 + 3) // 4)
    assert tiles >= 3 * SMS
    u, k, w, v = _inputs(B, H, N, "bf16", gated=True, seed=7)
    keep = 0xF000000F
    y, _, _ = _run(u, k, w, v, keep, "bf16")
    ref = oracle.fftconv_bins(u, k, W.monarch_binmask(keep, N), w=w, v=v)
    e = assert_close(y, ref, "bf16", f"monarch {tiles} tiles")
    print(f"monarch {tiles} tiles: rel_l2={e:.2e} max_abs={np.max(np.abs(y - ref)):.3e}")


def test_monarch_all_kept_equals_the_plain_forward():
    import torch
    B, H, N = 5, 3, 4096
    u, k, w, v = _inputs(B, H, N, "bf16", gated=True, seed=11)
    y, plan, Kf = _run(u, k, w, v, 0xFFFFFFFF, "bf16")
    y2 = plan.forward(to_dev(u, "bf16"), Kf, w=to_dev(w, "bf16"), v=to_dev(v, "bf16"))
    torch.cuda.synchronize()
    assert np.array_equal(y, y2.float().cpu().numpy().astype(np.float64))


def test_monarch_dc_only_and_empty_keep():
    """keep = {c2 = 0}: with the mirror rule only the eight bins f = 1024 c3
    survive (the mirror of c1 > 0, c2 = 0 has c2 = 31); keep = 0 gives y = 0."""
    import torch
    B, H, N = 2, 2, 4096
    u, k, w, v = _inputs(B, H, N, "f16", gated=False, seed=13)
    y, plan, Kf = _run(u, k, None, None, 0x1, "f16")
    assert_close(y, oracle.fftconv_bins(u, k, W.monarch_binmask(0x1, N)), "f16", "keep c2 = 0")
    y0 = plan.forward_monarch(to_dev(u, "f16"), Kf, 0)
    torch.cuda.synchronize()
    assert float(y0.abs().max()) == 0.0


def test_monarch_unsupported_plans():
    import torch
    import long_sequence_fft_b200 as lsf
    for N, order in ((1024, 0), (8192, 0), (4096, 1)):
        plan = lsf.Plan(N, 2, "bf16", order=order)
        Kf = plan.precompute(torch.zeros((2, N), dtype=torch.bfloat16, device="cuda"))
        u = torch.zeros((2, 2, N), dtype=torch.bfloat16, device="cuda")
        with pytest.raises(lsf.FFTConvError) as e:
            plan.forward_monarch(u, Kf, 0xF000000F)
        assert e.value.status == lsf.ERR_UNSUPPORTED


@pytest.mark.parametrize("B,H", [(1, 1), (3, 1), (2, 5)])
def test_monarch_small_and_ragged(B, H):
    N, keep = 4096, 0xF000000F
    u, k, w, v = _inputs(B, H, N, "f16", gated=True, seed=B * 10 + H)
    y, _, _ = _run(u, k, w, v, keep, "f16")
    assert_close(y, oracle.fftconv_bins(u, k, W.monarch_binmask(keep, N), w=w, v=v), "f16", f"monarch B={B} H={H}")
