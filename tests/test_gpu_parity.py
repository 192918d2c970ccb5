"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the
same seeded, dtype-rounded inputs.

Element-by-element at sizes the oracle finishes in seconds (several tiles and
ragged batches: odd B leaves an unpaired sequence), and on sampled outputs at
the workloads' full sizes, in the launch configuration the benchmark times."""
import numpy as np
import pytest

import oracle
import workloads as W
from parity_util import assert_close, rel_l2, run_cuda, to_dev

pytestmark = pytest.mark.gpu

RNG = np.random.default_rng(2024)


def _rand_inputs(B, H, N, L, dtype, gated, mask_frac=0.0, seed=0):
    rng = np.random.default_rng(seed)
    u = W.round_to(rng.standard_normal((B, H, N), dtype=np.float32), dtype)
    k = W.round_to((rng.standard_normal((H, L), dtype=np.float32) / np.float32(np.sqrt(L))), dtype)
    out = {"u": u, "k": k, "w": None, "v": None, "mask": None}
    if gated:
        out["w"] = W.round_to(rng.standard_normal((B, H, N), dtype=np.float32), dtype)
        out["v"] = W.round_to(rng.standard_normal((B, H, N), dtype=np.float32), dtype)
    if mask_frac > 0:
        m = (rng.random((H, N // 32)) >= mask_frac).astype(np.uint8)
        out["mask"] = m
    return out


def _oracle(inp):
    return oracle.fftconv(inp["u"], inp["k"], w=inp["w"], v=inp["v"], mask=inp["mask"])


# ------------------------------------------------------ small, full compare ---

CASES = []
for dtype in ("f32", "f16", "bf16"):
    for order in (1, 4, 0):
        for (B, H, N) in ((1, 2, 256), (3, 2, 1024), (2, 3, 4096), (1, 1, 8192)):
            CASES.append((dtype, order, B, H, N))
    CASES.append((dtype, 4, 2, 2, 16384))
    CASES.append((dtype, 0, 3, 2, 16384))
    CASES.append((dtype, 0, 3, 1, 32768))


@pytest.mark.parametrize("dtype,order,B,H,N", CASES)
def test_small_shapes_full_compare(dtype, order, B, H, N):
    inp = _rand_inputs(B, H, N, N, dtype, gated=(B % 2 == 1), seed=B * 131 + H * 7 + N)
    y, plan = run_cuda(inp, dtype, order=order)
    ref = _oracle(inp)
    assert_close(y, ref, dtype, f"{dtype} order={order} path={plan.path_name} B={B} H={H} N={N}")


@pytest.mark.parametrize("N", [2048, 4096])
@pytest.mark.parametrize("order", [1, 4, 0])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_partial_and_masked(order, dtype, N):
    import long_sequence_fft_b200 as lsf
    inp = _rand_inputs(3, 2, N, 300, dtype, gated=True, seed=7)
    y, _ = run_cuda(inp, dtype, order=order)
    assert_close(y, _oracle(inp), dtype, "partial L=300")
    inp = _rand_inputs(2, 3, N, N, dtype, gated=True, mask_frac=0.75, seed=8)
    if dtype != "f32" and order == 0 and N < 4096:
        # the tensor-core plan packs 4096 / N sequences into each transform
        # and has no 2N-point spectrum to mask: masks need order 1 or 4
        with pytest.raises(lsf.FFTConvError) as ei:
            run_cuda(inp, dtype, order=order)
        assert ei.value.status == lsf.ERR_UNSUPPORTED
        order = 1
    y, _ = run_cuda(inp, dtype, order=order)
    assert_close(y, _oracle(inp), dtype, "masked per-channel")
    inp["mask"] = inp["mask"][:1]
    y, _ = run_cuda(inp, dtype, order=order)
    assert_close(y, _oracle(inp), dtype, "masked shared row")


# ---------------------------------------------------------- workloads ---

REDUCED = {
    "fp32_n1k": dict(),                      # already small: full size
    "gated_bf16_n4k": dict(B=3, H=4),
    "fp16_n32k": dict(B=2, H=2),
    "dna_bf16_n1m": dict(H=2),
    "partial_bf16_n8k": dict(B=3, H=3),
    "sparse_bf16_n8k": dict(B=3, H=3),
    "dna_bf16_n4m_l1m": dict(H=2),
}


@pytest.mark.parametrize("name", sorted(REDUCED))
def test_workload_reduced_full_compare(name):
    w = W.WORKLOADS[name].with_shape(**REDUCED[name])
    inp = W.make_all(w)
    y, plan = run_cuda(inp, w.dtype)
    ref = _oracle(inp)
    assert_close(y, ref, w.dtype, f"{name} ({plan.path_name})")


def _sampled_ref(w, inp, seq, ts):
    if inp["mask"] is None:
        return oracle.direct_conv(inp["u"], inp["k"], w=inp["w"], v=inp["v"], seq=seq, ts=ts)
    # frequency-sparse: circular sum with the masked filter's time-domain
    # response, computed only for the channels that are sampled
    hs = np.unique(seq % w.H)
    keff = np.zeros((w.H, 2 * w.N))
    keff[hs] = oracle.masked_filter(inp["k"][hs], w.N, inp["mask"])
    return oracle.circular_conv_samples(inp["u"], keff, seq, ts, w=inp["w"], v=inp["v"])


@pytest.mark.parametrize("name", sorted(W.WORKLOADS))
def test_workload_full_size_sampled(name):
    """Full workload shapes, the benchmark's launch configuration (order 0),
    compared at seeded sample points against direct sums."""
    w = W.WORKLOADS[name]
    inp = W.make_all(w)
    y, plan = run_cuda(inp, w.dtype)
    seq, ts = W.sample_points(w, nseq=16, nrand=61)
    ref = _sampled_ref(w, inp, seq, ts)
    got = y.reshape(w.B * w.H, w.N)[seq, ts]
    assert_close(got, ref, w.dtype, f"{name} sampled ({plan.path_name})")
    # properties that hold at any size: finite everywhere
    assert np.isfinite(y).all()


# -------------------------------------------------------------- edges ---

def test_filter_export_matches_oracle_rfft():
    import long_sequence_fft_b200 as lsf
    for dtype, order, N, L in (("f32", 1, 1024, 1024), ("bf16", 4, 4096, 1000), ("f16", 0, 2048, 2048),
                               ("bf16", 0, 4096, 4096), ("f16", 0, 4096, 3000)):
        k = W.round_to(RNG.standard_normal((3, L), dtype=np.float32), dtype)
        plan = lsf.Plan(N, 3, dtype, order=order, L=L)
        Kf = plan.precompute(to_dev(k, dtype))
        got = plan.export_rfft(Kf).cpu().numpy().astype(np.complex128)
        ref = oracle.filter_rfft(k, N)
        err = np.linalg.norm(got - ref) / np.linalg.norm(ref)
        # fp32 spectra: 1e-5; the tensor-core path stores fp16 spectra with a
        # per-channel scale: 1e-3 relative (half-precision storage bound)
        tol = 1e-3 if plan.path_name == "tc_fused" else 1e-5
        assert err <= tol, (dtype, order, plan.path_name, err)


@pytest.mark.parametrize("order", [1, 4])
def test_delta_and_scalar_filters(order):
    import long_sequence_fft_b200 as lsf
    import torch
    N = 1024
    inp = _rand_inputs(3, 2, N, N, "f32", gated=True, seed=3)
    inp["k"] = np.zeros((2, N), np.float32)
    inp["k"][:, 0] = 1.0
    y, _ = run_cuda(inp, "f32", order=order)
    assert_close(y, inp["u"] * inp["w"] * inp["v"], "f32", "delta filter")
    # L = 1 partial filter
    inp["k"] = np.array([[2.0], [-0.5]], np.float32)
    y, _ = run_cuda(inp, "f32", order=order)
    ref = inp["u"] * inp["w"] * inp["v"] * inp["k"][None, :, :1]
    assert_close(y, ref, "f32", "L=1 filter")


@pytest.mark.parametrize("order", [1, 4])
def test_zero_and_full_masks(order):
    N = 1024
    inp = _rand_inputs(2, 2, N, N, "f32", gated=False, seed=5)
    inp["mask"] = np.zeros((1, N // 32), np.uint8)
    y, _ = run_cuda(inp, "f32", order=order)
    assert np.max(np.abs(y)) == 0.0
    inp["mask"] = np.full((2, N // 32), 7, np.uint8)     # any nonzero byte keeps
    y1, _ = run_cuda(inp, "f32", order=order)
    inp["mask"] = None
    y2, _ = run_cuda(inp, "f32", order=order)
    assert np.array_equal(y1, y2)


def test_empty_batch_is_noop():
    import long_sequence_fft_b200 as lsf
    import torch
    plan = lsf.Plan(1024, 2, "bf16")
    Kf = plan.precompute(torch.zeros((2, 1024), dtype=torch.bfloat16, device="cuda"))
    u = torch.zeros((0, 2, 1024), dtype=torch.bfloat16, device="cuda")
    y = plan.forward(u, Kf)
    assert y.shape == (0, 2, 1024)


def test_forward_host_matches_device_path():
    import long_sequence_fft_b200 as lsf
    import torch
    w = W.WORKLOADS["gated_bf16_n4k"].with_shape(B=3, H=5)
    inp = W.make_all(w)
    plan = lsf.Plan(w.N, w.H, "bf16")
    Kf = plan.precompute(to_dev(inp["k"], "bf16"))
    yd = plan.forward(to_dev(inp["u"], "bf16"), Kf, w=to_dev(inp["w"], "bf16"), v=to_dev(inp["v"], "bf16"))
    pin = lambda a: torch.from_numpy(a).to(torch.bfloat16).pin_memory()
    uh, wh, vh = pin(inp["u"]), pin(inp["w"]), pin(inp["v"])
    yh = torch.empty_like(uh).pin_memory()
    staging = torch.empty(plan.staging_bytes(w.B, True, True), dtype=torch.uint8, device="cuda")
    plan.forward_host(uh, Kf, yh, staging, w_host=wh, v_host=vh)
    torch.cuda.synchronize()
    assert torch.equal(yh, yd.cpu())


def test_bad_arguments_are_rejected_without_launch():
    import long_sequence_fft_b200 as lsf
    import torch
    plan = lsf.Plan(1024, 2, "f32")
    k = torch.zeros((2, 1024), device="cuda")
    Kf = plan.precompute(k)
    u = torch.zeros((2, 2, 1024), device="cuda")
    with pytest.raises(lsf.FFTConvError) as e:
        lib = lsf.library()
        rc = lib.fftconv_forward(plan.handle, u.data_ptr() + 4, Kf.data_ptr(), u.data_ptr() + 8192 * 4, 2, 2, 1024,
                                 None, None, None, 0, None)
        lsf._check(rc)
    assert e.value.status == lsf.ERR_ALIGNMENT
    with pytest.raises(lsf.FFTConvError) as e:
        lsf._check(lsf.library().fftconv_forward(plan.handle, u.data_ptr(), Kf.data_ptr(), u.data_ptr(), 2, 2,
                                                 1024, None, None, None, 0, None))
    assert e.value.status == lsf.ERR_INVALID_ARG        # y aliases u
    with pytest.raises(lsf.FFTConvError) as e:
        lsf._check(lsf.library().fftconv_forward(plan.handle, u.data_ptr(), Kf.data_ptr(), u.data_ptr(), 2, 3,
                                                 1024, None, None, None, 0, None))
    assert e.value.status == lsf.ERR_INVALID_ARG        # H mismatch
    with pytest.raises(lsf.FFTConvError) as e:
        lsf.Plan(1000, 2, "f32")
    assert e.value.status == lsf.ERR_UNSUPPORTED


# ------------------------------------------------- overlap-save windows ---

@pytest.mark.parametrize("dtype", ["bf16", "f16"])
@pytest.mark.parametrize("N,L,B", [(8192, 2048, 3), (8192, 2049, 2), (8192, 1, 1), (16384, 300, 3), (32768, 300, 3),
                                   (32768, 1024, 1)])
def test_overlap_save_windows(dtype, N, L, B):
    """Sequences longer than 4096 with filters of L <= 2049 taps run on the
    tensor-core kernel: as overlapping 4096-sample windows (N >= 32768) or as
    two or four blocks of 4096 (N = 8192, 16384)."""
    inp = _rand_inputs(B, 2, N, L, dtype, gated=(B != 1), seed=N + L + B)
    y, plan = run_cuda(inp, dtype, order=0)
    assert plan.path_name == "tc_fused"
    assert_close(y, _oracle(inp), dtype, f"overlap-save {dtype} N={N} L={L} B={B}")


def test_overlap_save_limits():
    import long_sequence_fft_b200 as lsf
    import torch
    # one tap too many for the windows: at N = 8192 and 16384 the block modes
    # (at 8192 with a mask, the parity split) serve it, longer sequences go to
    # the staged path
    assert lsf.Plan(8192, 2, "bf16", L=2050).path_name == "tc_fused"
    assert lsf.Plan(16384, 2, "bf16", L=2050).path_name == "tc_fused"
    assert lsf.Plan(32768, 2, "bf16", L=2050).path_name != "tc_fused"
    # windows (N = 32768) and four blocks (N = 16384) store 8192-point spectra
    # only: no block mask, no 2N-point export
    for N in (32768, 16384):
        plan = lsf.Plan(N, 2, "bf16", L=2048)
        assert plan.path_name == "tc_fused"
        k = torch.zeros((2, 2048), dtype=torch.bfloat16, device="cuda")
        Kf = plan.precompute(k)
        u = torch.zeros((2, 2, N), dtype=torch.bfloat16, device="cuda")
        mask = torch.ones((1, N // 32), dtype=torch.uint8, device="cuda")
        with pytest.raises(lsf.FFTConvError) as e:
            plan.forward(u, Kf, mask=mask)
        assert e.value.status == lsf.ERR_UNSUPPORTED
        with pytest.raises(lsf.FFTConvError) as e:
            plan.export_rfft(Kf)
        assert e.value.status == lsf.ERR_UNSUPPORTED


def test_forward_host_pipelined_chunks_match_device_path():
    """Odd B spread over several upload/compute/download chunks, with gates
    and a mask: bit-identical to the device-buffer call."""
    import long_sequence_fft_b200 as lsf
    import torch
    inp = _rand_inputs(19, 3, 2048, 2048, "bf16", gated=True, mask_frac=0.5, seed=11)
    plan = lsf.Plan(2048, 3, "bf16", order=1)         # (a masked plan at N < 4096: fp32 lanes)
    Kf = plan.precompute(to_dev(inp["k"], "bf16"))
    mask = torch.from_numpy(inp["mask"]).cuda()
    yd = plan.forward(to_dev(inp["u"], "bf16"), Kf, w=to_dev(inp["w"], "bf16"), v=to_dev(inp["v"], "bf16"),
                      mask=mask)
    pin = lambda a: torch.from_numpy(a).to(torch.bfloat16).pin_memory()
    uh, wh, vh = pin(inp["u"]), pin(inp["w"]), pin(inp["v"])
    mh = torch.from_numpy(inp["mask"]).pin_memory()
    yh = torch.empty_like(uh).pin_memory()
    staging = torch.empty(plan.staging_bytes(19, True, True, mh.shape[0]), dtype=torch.uint8, device="cuda")
    for _ in range(2):                                   # reuses the plan's copy streams
        yh.zero_()
        plan.forward_host(uh, Kf, yh, staging, w_host=wh, v_host=vh, mask_host=mh)
        torch.cuda.synchronize()
        assert torch.equal(yh, yd.cpu())


# ---------------------------------------------- N = 8192 parity split ---

@pytest.mark.parametrize("dtype", ["bf16", "f16"])
@pytest.mark.parametrize("B,L,gated,mask_frac", [(3, 8192, True, 0.0), (2, 8192, False, 0.75), (1, 5000, True, 0.5),
                                                 (5, 2050, True, 0.0), (4, 8192, True, 0.3)])
def test_split_n8192_full_filters(dtype, B, L, gated, mask_frac):
    """N = 8192 with any filter length: unmasked calls run the two-block mode,
    masked calls the 16384-point spectrum split by bin parity."""
    inp = _rand_inputs(B, 3, 8192, L, dtype, gated=gated, mask_frac=mask_frac, seed=B * 7 + L)
    y, plan = run_cuda(inp, dtype, order=0)
    assert plan.path_name == "tc_fused"
    assert_close(y, _oracle(inp), dtype, f"split {dtype} B={B} L={L} mask={mask_frac}")


def test_split_n8192_export_and_shared_mask():
    import long_sequence_fft_b200 as lsf
    k = W.round_to(RNG.standard_normal((3, 8192), dtype=np.float32) / 90.0, "bf16")
    plan = lsf.Plan(8192, 3, "bf16")
    Kf = plan.precompute(to_dev(k, "bf16"))
    got = plan.export_rfft(Kf).cpu().numpy().astype(np.complex128)
    ref = oracle.filter_rfft(k, 8192)
    assert np.linalg.norm(got - ref) / np.linalg.norm(ref) <= 1e-3
    inp = _rand_inputs(3, 3, 8192, 8192, "bf16", gated=True, mask_frac=0.75, seed=21)
    inp["mask"] = inp["mask"][:1]
    y, _ = run_cuda(inp, "bf16")
    assert_close(y, _oracle(inp), "bf16", "split, one mask row for all channels")


# ------------------------------------- staged path, tensor-core row pass ---

@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("N,L,B,H,gated,mask_frac", [
    (16384, 16384, 3, 2, True, 0.0),        # R = 4: one tile per pair, an unpaired row
    (16384, 2050, 4, 3, False, 0.5),        # shortest filter the staged tiles take
    (32768, 4096, 2, 3, True, 0.3),
    (65536, 65536, 1, 2, True, 0.0),        # R = 16: four tiles per pair
    (1 << 20, 1 << 20, 1, 5, False, 0.0),   # R = 256, 4 pairs per workspace chunk: 2 chunks
])
def test_tc_staged_rows(dtype, N, L, B, H, gated, mask_frac):
    """Long sequences on the staged path whose row pass (rows of 8192) runs
    on the tensor cores, against the oracle element by element."""
    inp = _rand_inputs(B, H, N, L, dtype, gated=gated, mask_frac=mask_frac, seed=N // 1024 + L + B)
    y, plan = run_cuda(inp, dtype, order=5)
    assert plan.path_name == "tc_staged"
    assert_close(y, _oracle(inp), dtype, f"tc_staged {dtype} N={N} L={L} B={B} H={H} mask={mask_frac}")


def test_tc_staged_is_the_automatic_choice_and_exports():
    import long_sequence_fft_b200 as lsf
    k = W.round_to(RNG.standard_normal((3, 32768), dtype=np.float32) / 180.0, "f16")
    plan = lsf.Plan(32768, 3, "f16")
    assert plan.path_name == "tc_staged"
    Kf = plan.precompute(to_dev(k, "f16"))
    got = plan.export_rfft(Kf).cpu().numpy().astype(np.complex128)
    ref = oracle.filter_rfft(k, 32768)
    # fp16 spectrum rows, each with its own scale: half-precision storage bound
    assert np.linalg.norm(got - ref) / np.linalg.norm(ref) <= 1e-3
    # the short-filter plan of the same length keeps the overlap-save windows
    assert lsf.Plan(32768, 3, "f16", L=2049).path_name == "tc_fused"
    # the SIMT staged path stays available as order 4
    assert lsf.Plan(32768, 3, "f16", order=4).path_name == "simt_staged"


def test_tc_staged_forward_host_chunks():
    """The pipelined host-buffer call splits the batch into chunks; each
    chunk's launches start at its own pair offset."""
    import torch
    import long_sequence_fft_b200 as lsf
    B, H, N = 9, 2, 16384
    inp = _rand_inputs(B, H, N, N, "bf16", gated=True, seed=99)
    plan = lsf.Plan(N, H, "bf16", order=5)
    Kf = plan.precompute(to_dev(inp["k"], "bf16"))
    tdt = W.torch_dtype("bf16")
    host = {n: torch.from_numpy(inp[n]).to(tdt).pin_memory() for n in ("u", "w", "v")}
    y_host = torch.empty((B, H, N), dtype=tdt).pin_memory()
    staging = torch.empty(plan.staging_bytes(B, True, True), dtype=torch.uint8, device="cuda")
    plan.forward_host(host["u"], Kf, y_host, staging, w_host=host["w"], v_host=host["v"])
    torch.cuda.synchronize()
    assert plan.device_status() == 0
    assert_close(y_host.float().numpy().astype(np.float64), _oracle(inp), "bf16", "tc_staged forward_host")


@pytest.mark.parametrize("dtype,order,N,L,B,H,gated,mask_frac", [
    ("f32", 4, 1 << 17, 1 << 17, 1, 2, False, 0.0),     # fp32 staged, 256 x 1024
    ("bf16", 4, 1 << 18, 5000, 3, 1, True, 0.5),        # 256 x 1024, partial filter, mask
    ("f16", 5, 1 << 21, 1 << 21, 1, 1, True, 0.0),      # tensor-core rows, 512 x 8192
    ("bf16", 5, 1 << 18, 1 << 18, 2, 2, False, 0.25),   # tensor-core rows, 64 x 8192
    ("bf16", 5, 1 << 22, 1 << 20, 1, 1, True, 0.5),     # 4M with a 1M filter: 1024 x 8192
    ("f32", 4, 1 << 22, 1 << 20, 1, 1, False, 0.0),     # the same on fp32 lanes, 512 x 16384
])
def test_staged_long_columns(dtype, order, N, L, B, H, gated, mask_frac):
    """Long columns (64 to 512 values: the shared-memory column passes) with
    fp32 and tensor-core row passes, against the oracle element by element."""
    inp = _rand_inputs(B, H, N, L, dtype, gated=gated, mask_frac=mask_frac, seed=N // 4096 + order)
    y, plan = run_cuda(inp, dtype, order=order)
    assert plan.path_name == ("simt_staged" if order == 4 else "tc_staged")
    assert_close(y, _oracle(inp), dtype, f"staged {dtype} order={order} N={N} L={L}")


@pytest.mark.parametrize("dtype,N,L,B,H,nwin", [
    ("bf16", 32768, 4096, 3, 2, 2),          # hop 16384: 32768-point windows, 4 x 8192
    ("f16", 65536, 16384, 2, 1, 4),          # L equal to the hop
    ("bf16", 1 << 20, 20000, 1, 2, 32),      # hop 32768: 8 x 8192 columns in registers
    ("f16", 1 << 21, 300000, 1, 1, 4),       # hop 2^19: 128 x 8192 columns in shared memory
])
def test_tc_staged_overlap_save_windows(dtype, N, L, B, H, nwin):
    """Automatic plans with a filter much shorter than the sequence run the
    staged tensor-core path over overlap-save windows (2 x hop points, the
    first window's first half zero, each window's second half output)."""
    inp = _rand_inputs(B, H, N, L, dtype, gated=True, seed=N // 1024 + L % 977)
    y, plan = run_cuda(inp, dtype, order=0)
    assert plan.path_name == "tc_staged"
    assert_close(y, _oracle(inp), dtype, f"tc_staged windows {dtype} N={N} L={L} B={B} (nwin={nwin})")
    # the same filter without windows (order 5) agrees with the oracle too
    y5, plan5 = run_cuda(inp, dtype, order=5)
    assert_close(y5, _oracle(inp), dtype, f"tc_staged full {dtype} N={N} L={L}")


def test_tc_staged_windows_reject_mask_and_export():
    import torch
    import long_sequence_fft_b200 as lsf
    N, H, L = 32768, 2, 4096
    inp = _rand_inputs(1, H, N, L, "bf16", gated=False, mask_frac=0.5, seed=5)
    plan = lsf.Plan(N, H, "bf16", L=L)
    Kf = plan.precompute(to_dev(inp["k"], "bf16"))
    u = to_dev(inp["u"], "bf16")
    with pytest.raises(lsf.FFTConvError) as ei:
        plan.forward(u, Kf, mask=torch.from_numpy(inp["mask"]).cuda())
    assert ei.value.status == lsf.ERR_UNSUPPORTED
    with pytest.raises(lsf.FFTConvError) as ei:
        plan.export_rfft(Kf)
    assert ei.value.status == lsf.ERR_UNSUPPORTED
    assert plan.device_status() == 0
