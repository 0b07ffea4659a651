"""GPU parity: the CUDA path through the C ABI against the fp64 CPU oracle.

Small problems (several chunks, ragged tails, every output dtype) are compared element by
element; the four prefill workloads run at full size in the launch configuration the
benchmark times, and are compared on sampled (batch, head) pairs, whole sequences, which the
oracle computes one by one.  ChunkBMM tiles must be bit-exact.
"""
import numpy as np
import pytest
import torch

import oracle
from quantized_mamba_ssd_b200 import build as qbuild
from quantized_mamba_ssd_b200 import ssd_i8
from quantized_mamba_ssd_b200 import workloads as W
from parity_util import REL_L2, check_close, check_i8, head_subset

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    qbuild.build()
    ssd_i8.library()


def mk(b, L, H, G, N, Q, **kw):
    """A prefill case with headdim 64, sizes given as (batch, seqlen, heads, groups, dstate,
    chunk)."""
    return W.make_prefill(b, L, H, 64, N, G, Q, **kw)


def dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.to(dtype)
    return t.to(DEV)


def gpu_scan(case, y_dtype="f32", y_scale=1.0, chunk_size=None, init=True, final=True):
    bsz, L, H, P, N = case.batch, case.seqlen, case.nheads, case.headdim, case.dstate
    fs = torch.empty((bsz, H, P, N), dtype=torch.float32, device=DEV) if final else None
    y = ssd_i8.ssd_i8_chunk_scan(
        dev(case.x), dev(case.B), dev(case.C), dev(case.dt), dev(case.A), dev(case.D),
        dev(case.x_scale), dev(case.B_scale), dev(case.C_scale),
        chunk_size or case.chunk_size,
        init_state=dev(case.init_state) if (init and case.init_state is not None) else None,
        final_state=fs, y_dtype=y_dtype, y_scale=y_scale)
    torch.cuda.synchronize()
    return y.cpu().numpy(), (fs.cpu().numpy() if final else None)


def oracle_scan(case, **kw):
    return oracle.scan(case.x, case.B, case.C, case.dt, case.A, case.D, case.x_scale,
                       case.B_scale, case.C_scale, init_state=case.init_state, **kw)[:2]


SMALL = [
    # b, L, H, G, N, Q, law, scales, init, out
    (2, 300, 8, 2, 128, 64, "laplace_outliers_all", "head", True, "f32"),
    (2, 300, 8, 2, 128, 128, "laplace_outliers_all", "head", True, "f16"),
    (1, 517, 4, 4, 128, 256, "laplace_spread", "head", True, "f32"),
    (3, 200, 6, 3, 16, 64, "normal", "tensor", False, "f16"),
    (2, 130, 4, 1, 32, 128, "laplace_outliers_x", "head", True, "f32"),
    (2, 257, 4, 2, 64, 256, "laplace_outliers_all", "head", False, "f16"),
    (1, 1, 4, 2, 128, 256, "normal", "head", True, "f32"),
    (1, 63, 2, 1, 128, 64, "normal", "head", True, "f32"),
    # per-tensor static scales with x clipped at the 99.99th percentile (saturated codes)
    (2, 600, 8, 2, 128, 256, "laplace_outliers_all", "percentile", True, "f32"),
    (1, 300, 4, 1, 64, 128, "laplace_outliers_x", "percentile", False, "f16"),
]


@pytest.mark.parametrize("b,L,H,G,N,Q,law,scales,init,out", SMALL)
def test_small_prefill_matches_oracle(b, L, H, G, N, Q, law, scales, init, out):
    case = W.make_prefill(b, L, H, 64, N, G, Q, law=law, scales=scales, seed=L + H + N,
                          with_init_state=init)
    y, fs = gpu_scan(case, y_dtype=out)
    yr, fr = oracle_scan(case)
    check_close(y, yr, "y")
    check_close(fs, fr, "final_state")


@pytest.mark.parametrize("Q", [64, 256])
def test_small_prefill_int8_output(Q):
    case = mk(2, 400, 8, 2, 128, Q, law="laplace_outliers_all", scales="head",
                          seed=77, with_init_state=True)
    yr, _ = oracle_scan(case)
    s_y = float(np.abs(yr).max() / 127.0)
    yq, _ = gpu_scan(case, y_dtype="i8", y_scale=s_y)
    check_i8(yq, oracle.requant(yr, s_y))


def test_int8_output_is_the_fp32_output_requantized():
    # the int8 epilogue must be q = clamp(rint(y * fp32(1/s_y))) of the very y the f32 path
    # writes, the product taken exactly (fp64 holds the product of two fp32 values) and rounded
    # once
    case = mk(1, 333, 4, 2, 128, 128, law="laplace_outliers_all", seed=5)
    y32, _ = gpu_scan(case, y_dtype="f32")
    s_y = np.float32(np.abs(y32).max() / 100.0)
    yq, _ = gpu_scan(case, y_dtype="i8", y_scale=float(s_y))
    inv = np.float32(1.0) / s_y
    ref = np.clip(np.rint(y32.astype(np.float64) * np.float64(inv)), -127, 127).astype(np.int8)
    assert np.array_equal(yq, ref)


def test_int8_rounding_rule_at_full_size():
    """The 8B-shaped prefill with s_y = 0.05: at this size some products y * fp32(1/s_y) fall
    close enough to a half-integer that rounding them to fp32 first would move the code.  The
    epilogue rounds the exact product once, in every one of the 2^28 outputs."""
    case = W.make_prefill_config(3)
    y32, _ = gpu_scan(case, y_dtype="f32", init=False, final=False)
    yq, _ = gpu_scan(case, y_dtype="i8", y_scale=0.05, init=False, final=False)
    inv = np.float32(1.0) / np.float32(0.05)
    once = twice = 0
    flat32, flatq = y32.reshape(-1, 1 << 20), yq.reshape(-1, 1 << 20)
    for a, q in zip(flat32, flatq):
        ref1 = np.clip(np.rint(a.astype(np.float64) * np.float64(inv)), -127, 127).astype(np.int8)
        ref2 = np.clip(np.rint(a * inv), -127, 127).astype(np.int8)   # fp32 product first
        once += int((q != ref1).sum())
        twice += int((ref1 != ref2).sum())
    assert once == 0, f"{once} int8 outputs differ from the one-rounding rule"
    assert twice > 0, "no output distinguishes the two roundings: the check has no power here"


# ---------------------------------------------------------------------------------------
# the four prefill workloads at full size, sampled (batch, head) pairs
# ---------------------------------------------------------------------------------------
SAMPLES = {0: None, 1: [(0, 0), (3, 63), (1, 17), (2, 40)],
           2: [(0, 0), (7, 79), (3, 33), (5, 61)],
           3: [(0, 0), (1, 127), (0, 77), (1, 35), (0, 16), (1, 100)],
           4: [(0, 5), (1, 126), (0, 64), (1, 31)]}


def _compare_sampled(case, y, fs, pairs, out):
    for b, h in pairs:
        sub = head_subset(case, [h], batches=[b])
        yr, fr, _ = oracle.scan(**sub)
        if out == "i8":
            continue
        check_close(y[b, :, h, :], yr[0, :, 0, :], f"y[b={b},h={h}]")
        check_close(fs[b, h], fr[0, 0], f"final_state[b={b},h={h}]")


@pytest.mark.parametrize("cfg", [0, 1, 2, 3, 4])
def test_workload_prefill_matches_oracle(cfg):
    case = W.make_prefill_config(cfg)
    out = case.out_dtype
    pairs = SAMPLES[cfg]
    if pairs is None:  # tiny workload: the oracle does all of it
        y, fs = gpu_scan(case, y_dtype=out)
        yr, fr = oracle_scan(case)
        check_close(y, yr, "y")
        check_close(fs, fr, "final_state")
        return
    if out == "i8":
        # calibrate the static output scale on the oracle's sampled outputs, then check the
        # requantized output and the f32 output of the same launch configuration
        refs = {}
        for b, h in pairs:
            yr, fr, _ = oracle.scan(**head_subset(case, [h], batches=[b]))
            refs[(b, h)] = (yr[0, :, 0, :], fr[0, 0])
        s_y = float(max(np.abs(r[0]).max() for r in refs.values()) / 127.0)
        yq, fs = gpu_scan(case, y_dtype="i8", y_scale=s_y)
        for (b, h), (yr, fr) in refs.items():
            check_i8(yq[b, :, h, :], oracle.requant(yr, s_y))
            check_close(fs[b, h], fr, f"final_state[b={b},h={h}]")
        y32, _ = gpu_scan(case, y_dtype="f32", final=False)
        for (b, h), (yr, _) in refs.items():
            check_close(y32[b, :, h, :], yr, f"y[b={b},h={h}]")
        return
    y, fs = gpu_scan(case, y_dtype=out)
    _compare_sampled(case, y, fs, pairs, out)


def test_long_prefill_keeps_half_the_error_margin():
    # The non-int8 MMA operands are rounded to f16 once each (a design choice, not the pages'
    # hi/lo int8 split).  This guards the margin that leaves on the 8B-shaped workload: the f32
    # output of sampled whole (batch, head) sequences within half the relative-L2 tolerance.
    case = W.make_prefill_config(3)
    y32, _ = gpu_scan(case, y_dtype="f32", final=False)
    for b, h in SAMPLES[3][:4]:
        yr, _, _ = oracle.scan(**head_subset(case, [h], batches=[b]))
        ref = yr[0, :, 0, :]
        rel = np.linalg.norm(y32[b, :, h, :] - ref) / np.linalg.norm(ref)
        assert rel <= 0.5 * REL_L2, f"y[b={b},h={h}]: rel-L2 {rel:.3e} above half the tolerance"


# ---------------------------------------------------------------------------------------
# ChunkBMM: exact int32
# ---------------------------------------------------------------------------------------
@pytest.mark.parametrize("L,G,N,Q", [(300, 2, 128, 64), (517, 1, 128, 256), (200, 3, 16, 64),
                                     (130, 2, 32, 128), (257, 2, 64, 256)])
def test_chunk_cb_bit_exact(L, G, N, Q):
    rng = np.random.default_rng(L * N)
    C = rng.integers(-127, 128, size=(2, L, G, N), dtype=np.int8)
    B = rng.integers(-127, 128, size=(2, L, G, N), dtype=np.int8)
    cb = ssd_i8.ssd_i8_chunk_cb(dev(C), dev(B), Q)
    torch.cuda.synchronize()
    assert np.array_equal(cb.cpu().numpy().astype(np.int64), oracle.chunk_cb(C, B, Q))


def test_chunk_cb_bit_exact_at_workload_size():
    case = W.make_prefill_config(3)
    Q = case.chunk_size
    cb = ssd_i8.ssd_i8_chunk_cb(dev(case.C), dev(case.B), Q).cpu().numpy()
    for b, c in [(0, 0), (1, 63), (0, 31), (1, 7)]:
        sl = slice(c * Q, (c + 1) * Q)
        ref = oracle.chunk_cb(case.C[b:b + 1, sl], case.B[b:b + 1, sl], Q)
        assert np.array_equal(cb[b, c].astype(np.int64), ref[0, 0])


# ---------------------------------------------------------------------------------------
# invariants and edge cases
# ---------------------------------------------------------------------------------------
def test_chunk_size_does_not_change_the_result():
    case = mk(2, 700, 4, 2, 128, 64, law="laplace_outliers_all", seed=9,
                          with_init_state=True)
    ys = [gpu_scan(case, chunk_size=q) for q in (64, 128, 256)]
    yr, fr = oracle_scan(case)
    for y, fs in ys:
        check_close(y, yr)
        check_close(fs, fr, "final_state")
    check_close(ys[0][0], ys[2][0], "Q=64 vs Q=256")


@pytest.mark.parametrize("split", [200, 256])
def test_split_prefill_hands_state_on(split):
    case = mk(2, 600, 4, 2, 128, 128, law="laplace_outliers_all", seed=10,
                          with_init_state=True)
    y, fs = gpu_scan(case)
    import copy
    a = copy.copy(case)
    a.x, a.B, a.C, a.dt, a.seqlen = case.x[:, :split], case.B[:, :split], case.C[:, :split], \
        case.dt[:, :split], split
    y1, f1 = gpu_scan(a)
    bcase = copy.copy(case)
    bcase.x, bcase.B, bcase.C, bcase.dt, bcase.seqlen = case.x[:, split:], case.B[:, split:], \
        case.C[:, split:], case.dt[:, split:], case.seqlen - split
    bcase.init_state = f1
    y2, f2 = gpu_scan(bcase)
    check_close(np.concatenate([y1, y2], axis=1), y, "split y")
    check_close(f2, fs, "split final_state")


def test_decode_step_equals_length_one_prefill():
    d = W.make_decode(4, 1, 8, 64, 128, 2, seed=12)
    st = dev(d.state)
    y_dec = ssd_i8.ssd_i8_state_update(st, dev(d.x[0]), dev(d.B[0]), dev(d.C[0]), dev(d.dt[0]),
                                       dev(d.A), dev(d.D), dev(d.x_scale), dev(d.B_scale),
                                       dev(d.C_scale), y_dtype="f32")
    case = W.PrefillCase("L1", 4, 1, 8, 64, 128, 2, 64, d.x[0][:, None], d.B[0][:, None],
                         d.C[0][:, None], d.dt[0][:, None], d.A, d.D, d.x_scale, d.B_scale,
                         d.C_scale, "f32", d.state)
    y_pf, fs = gpu_scan(case)
    check_close(y_dec.cpu().numpy(), y_pf[:, 0], "decode vs L=1 prefill")
    check_close(st.cpu().numpy(), fs, "decode state vs L=1 prefill")


def test_deterministic():
    case = mk(2, 513, 8, 2, 128, 256, law="laplace_outliers_all", seed=13,
                          with_init_state=True)
    y1, f1 = gpu_scan(case)
    y2, f2 = gpu_scan(case)
    assert np.array_equal(y1, y2) and np.array_equal(f1, f2)


def test_empty_sequence_copies_initial_state():
    case = mk(2, 8, 4, 2, 128, 64, seed=14, with_init_state=True)
    fs = torch.full((2, 4, 64, 128), 7.0, device=DEV)
    z8 = torch.empty((2, 0, 4, 64), dtype=torch.int8, device=DEV)
    zb = torch.empty((2, 0, 2, 128), dtype=torch.int8, device=DEV)
    y = ssd_i8.ssd_i8_chunk_scan(z8, zb, zb, torch.empty((2, 0, 4), device=DEV), dev(case.A),
                                 dev(case.D), dev(case.x_scale), dev(case.B_scale),
                                 dev(case.C_scale), 64, init_state=dev(case.init_state),
                                 final_state=fs, y_dtype="f32")
    torch.cuda.synchronize()
    assert y.numel() == 0
    assert np.array_equal(fs.cpu().numpy(), case.init_state)


def test_special_inputs_zero_dt_and_strong_decay():
    case = mk(1, 300, 4, 2, 128, 128, seed=15, with_init_state=True)
    case.dt[:, :100] = 0.0   # no update: state carries over unchanged
    case.dt[:, 200:] = 6.0   # exp(dt A) underflows towards zero
    y, fs = gpu_scan(case)
    yr, fr = oracle_scan(case)
    check_close(y, yr)
    check_close(fs, fr, "final_state")


def test_status_query_after_a_clean_call():
    case = mk(2, 300, 8, 2, 128, 64, seed=18, with_init_state=True)
    ws = torch.empty(ssd_i8.ssd_i8_chunk_scan_workspace_size(2, 300, 8, 64, 128, 2, 64),
                     dtype=torch.uint8, device=DEV)
    ssd_i8.ssd_i8_chunk_scan(dev(case.x), dev(case.B), dev(case.C), dev(case.dt), dev(case.A),
                             dev(case.D), dev(case.x_scale), dev(case.B_scale), dev(case.C_scale),
                             64, workspace=ws)
    ssd_i8.ssd_i8_chunk_scan_status(ws)  # raises on a device-side timeout


@pytest.mark.parametrize("b,L,H,G,Q", [(1, 4096, 2, 1, 256), (3, 1000, 50, 5, 128),
                                       (1, 64 * 300, 1, 1, 64)])
def test_range_split_hand_offs(b, L, H, G, Q):
    # work lists whose per-CTA ranges split sequences mid-way (one unit over many CTAs, and
    # ranges covering several units) exercise the state hand-off between CTAs
    case = mk(b, L, H, G, 128, Q, law="laplace_outliers_all", seed=L + H, with_init_state=True)
    y, fs = gpu_scan(case)
    pairs = [(0, 0), (b - 1, H - 1)]
    for bb, hh in pairs:
        yr, fr, _ = oracle.scan(**head_subset(case, [hh], batches=[bb]))
        check_close(y[bb, :, hh, :], yr[0, :, 0, :], f"y[b={bb},h={hh}]")
        check_close(fs[bb, hh], fr[0, 0], f"final_state[b={bb},h={hh}]")


def test_workspace_too_small_is_reported():
    case = mk(1, 100, 4, 2, 128, 64, seed=16)
    with pytest.raises(ssd_i8.SSDError) as ei:
        ssd_i8.ssd_i8_chunk_scan(dev(case.x), dev(case.B), dev(case.C), dev(case.dt), dev(case.A),
                                 dev(case.D), dev(case.x_scale), dev(case.B_scale),
                                 dev(case.C_scale), 64,
                                 workspace=torch.empty(256, dtype=torch.uint8, device=DEV))
    assert ei.value.status == 3


# ---------------------------------------------------------------------------------------
# decode state update
# ---------------------------------------------------------------------------------------
@pytest.mark.parametrize("N,G,out", [(128, 2, "f32"), (16, 1, "f16"), (256, 4, "f32"),
                                     (64, 8, "f16")])
def test_decode_steps_match_oracle(N, G, out):
    d = W.make_decode(3, 5, 8, 64, N, G, seed=N + G)
    st = dev(d.state)
    ref_state = d.state.astype(np.float64)
    for s in range(d.steps):
        y = ssd_i8.ssd_i8_state_update(st, dev(d.x[s]), dev(d.B[s]), dev(d.C[s]), dev(d.dt[s]),
                                       dev(d.A), dev(d.D), dev(d.x_scale), dev(d.B_scale),
                                       dev(d.C_scale), y_dtype=out)
        yr = oracle.step(ref_state, d.x[s], d.B[s], d.C[s], d.dt[s], d.A, d.D, d.x_scale,
                         d.B_scale, d.C_scale)
        check_close(y.float().cpu().numpy(), yr, f"y step {s}")
    check_close(st.cpu().numpy(), ref_state, "state")


def test_decode_odd_headdim():
    d = W.make_decode(2, 3, 4, 40, 128, 2, seed=3)
    st = dev(d.state)
    ref_state = d.state.astype(np.float64)
    for s in range(d.steps):
        y = ssd_i8.ssd_i8_state_update(st, dev(d.x[s]), dev(d.B[s]), dev(d.C[s]), dev(d.dt[s]),
                                       dev(d.A), dev(d.D), dev(d.x_scale), dev(d.B_scale),
                                       dev(d.C_scale), y_dtype="f32")
        yr = oracle.step(ref_state, d.x[s], d.B[s], d.C[s], d.dt[s], d.A, d.D, d.x_scale,
                         d.B_scale, d.C_scale)
        check_close(y.cpu().numpy(), yr, f"y step {s}")
    check_close(st.cpu().numpy(), ref_state, "state")


def test_decode_workload_sampled():
    """The 512-step, batch-128 decode run at full size; sampled (batch, head) pairs through
    every step against the oracle."""
    d = W.make_decode_config()
    st = dev(d.state)
    pairs = [(0, 0), (127, 127), (64, 3), (5, 90)]
    ys = {p: [] for p in pairs}
    args = [dev(d.A), dev(d.D), dev(d.x_scale), dev(d.B_scale), dev(d.C_scale)]
    xs, Bs, Cs, dts = dev(d.x), dev(d.B), dev(d.C), dev(d.dt)
    for s in range(d.steps):
        y = ssd_i8.ssd_i8_state_update(st, xs[s], Bs[s], Cs[s], dts[s], *args, y_dtype="f16")
        for (b, h) in pairs:
            ys[(b, h)].append(y[b, h])
    final = st.cpu().numpy()
    H, G = d.nheads, d.ngroups
    for (b, h) in pairs:
        g = h // (H // G)
        ref = d.state[b:b + 1, h:h + 1].astype(np.float64).copy()
        got = torch.stack(ys[(b, h)]).float().cpu().numpy()
        refs = []
        for s in range(d.steps):
            refs.append(oracle.step(ref, d.x[s][b:b + 1, h:h + 1], d.B[s][b:b + 1, g:g + 1],
                                    d.C[s][b:b + 1, g:g + 1], d.dt[s][b:b + 1, h:h + 1],
                                    d.A[h:h + 1], d.D[h:h + 1], d.x_scale[h:h + 1],
                                    d.B_scale[g:g + 1], d.C_scale[g:g + 1])[0, 0])
        check_close(got, np.stack(refs), f"decode y (b={b}, h={h})")
        check_close(final[b, h], ref[0, 0], f"decode state (b={b}, h={h})")


def test_launch_count_claim():
    """The benchmark reports KERNELS_PER_CHUNK_SCAN launches per call; count them."""
    from torch.profiler import ProfilerActivity, profile
    case = mk(1, 300, 4, 2, 128, 128, seed=17)
    ins = [dev(a) for a in (case.x, case.B, case.C, case.dt, case.A, case.D, case.x_scale,
                            case.B_scale, case.C_scale)]
    y = torch.empty((1, 300, 4, 64), dtype=torch.float16, device=DEV)
    ws = torch.empty(ssd_i8.ssd_i8_chunk_scan_workspace_size(1, 300, 4, 64, 128, 2, 128),
                     dtype=torch.uint8, device=DEV)
    ssd_i8.ssd_i8_chunk_scan(*ins, 128, y=y, workspace=ws)
    torch.cuda.synchronize()
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        ssd_i8.ssd_i8_chunk_scan(*ins, 128, y=y, workspace=ws)
        torch.cuda.synchronize()
    kernels = [e.name for e in prof.events()
               if e.device_type == torch.autograd.DeviceType.CUDA
               and "Memcpy" not in e.name and "Memset" not in e.name]
    assert len(kernels) == ssd_i8.KERNELS_PER_CHUNK_SCAN, kernels
