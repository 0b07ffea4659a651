"""Exact readout of the chunk scan: on an input family where every intermediate is exactly
representable, the CUDA path must equal the fp64 oracle bit for bit, and y reads out the
ChunkBMM products C_t . B_s of the fused kernel one by one.

The family (``workloads.make_exact_readout``): B, C codes in {-1, 0, 1}; x one-hot, head j of a
group carrying token 64 j + p in column p; dt = 2^-3; A = D = 0; power-of-two scales.  The SSM
recurrence of the Mamba-2 SSD (the SSDi8 page, the state path and ChunkScan of Table 5; the
Ternary Mamba page, section 1) then gives y[b, t, h, p] = dt s_x s_B s_C (C_t . B_s) for
s = 64 j + p <= t and 0 for s > t: within a 128-token block this is the fused kernel's own
ChunkBMM times the causal mask; across blocks it is the state path (C_t . H with H built from
earlier blocks, handed between CTAs).  Every M', B', C', H' value the kernel rounds to f16 is a
small integer times a power of two, so nothing is rounded and the result must be exact.
"""
import numpy as np
import pytest
import torch

import oracle
from quantized_mamba_ssd_b200 import build as qbuild
from quantized_mamba_ssd_b200 import ssd_i8
from quantized_mamba_ssd_b200 import workloads as W

DEV = "cuda:0"

# b, L, G, N, Q, initial state
CASES = [
    (2, 320, 1, 128, 256, False),   # 5 heads, ragged last block
    (3, 200, 1, 16, 128, False),    # dstate 16, ragged
    (1, 256, 2, 64, 64, False),     # two groups
    (2, 300, 2, 128, 256, True),    # with an exactly representable initial state
    (1, 4096, 1, 128, 256, False),  # 64 heads x 32 blocks: blocks of one head on several CTAs
]


def _scale(case) -> float:
    return float(case.dt[0, 0, 0]) * float(case.x_scale[0]) * float(case.B_scale[0]) * \
        float(case.C_scale[0])


def _init_state(case, seed: int) -> np.ndarray:
    """Initial state with entries k / 8, k in {-2..2}: in units of s_x s_B = 1/8 an integer."""
    rng = np.random.default_rng(seed)
    k = rng.integers(-2, 3, size=(case.batch, case.nheads, case.headdim, case.dstate))
    return (k / 8.0).astype(np.float32)


def _closed_form(case, init) -> np.ndarray:
    """y from the closed form: dt s_x s_B s_C (C_t . B_s) for s = 64 j + p <= t, plus C_t . h0[p]
    s_C for an initial state h0 (A = 0: it never decays); exact integer products in int64."""
    b, L, H, P, G = case.batch, case.seqlen, case.nheads, case.headdim, case.ngroups
    per_group = H // G
    C64 = case.C.astype(np.int64)
    B64 = case.B.astype(np.int64)
    y = np.zeros((b, L, H, P), dtype=np.float64)
    t = np.arange(L)
    for g in range(G):
        CB = np.einsum("btn,bsn->bts", C64[:, :, g], B64[:, :, g])  # [b, t, s], exact
        for j in range(per_group):
            h = g * per_group + j
            s = P * j + np.arange(P)
            ok = s < L
            blk = np.zeros((b, L, P), dtype=np.int64)
            blk[:, :, ok] = CB[:, :, s[ok]]
            blk = np.where(t[None, :, None] >= s[None, None, :], blk, 0)
            y[:, :, h, :] = _scale(case) * blk
            if init is not None:
                y[:, :, h, :] += float(case.C_scale[g]) * np.einsum(
                    "btn,bpn->btp", C64[:, :, g].astype(np.float64), init[:, h].astype(np.float64))
    return y


@pytest.mark.parametrize("b,L,G,N,Q,init", CASES[:4])
def test_oracle_equals_the_closed_form(b, L, G, N, Q, init):
    """CPU: the oracle on this family is the closed form, exactly (a pin of the family itself,
    and of the oracle's causal sum and state path)."""
    case = W.make_exact_readout(b, L, G, N, Q, seed=L + N)
    h0 = _init_state(case, L) if init else None
    y, fs = oracle.scan(case.x, case.B, case.C, case.dt, case.A, case.D, case.x_scale,
                        case.B_scale, case.C_scale, init_state=h0)[:2]
    assert np.array_equal(y, _closed_form(case, h0))
    # final state: h0 + dt s_x s_B B_s for the one token s of each (head, column)
    ref = np.zeros_like(fs) if h0 is None else h0.astype(np.float64).copy()
    P = case.headdim
    per_group = case.nheads // G
    for h in range(case.nheads):
        g, j = divmod(h, per_group)
        for p in range(P):
            s = P * j + p
            if s < L:
                ref[:, h, p, :] += float(case.dt[0, 0, 0]) * float(case.x_scale[h]) * \
                    float(case.B_scale[g]) * case.B[:, s, g, :].astype(np.float64)
    assert np.array_equal(fs, ref)


@pytest.fixture(scope="module")
def _lib():
    qbuild.build()
    ssd_i8.library()


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def _gpu(case, h0, y_dtype, y_scale=1.0, hadamard=False):
    fs = torch.empty((case.batch, case.nheads, case.headdim, case.dstate), dtype=torch.float32,
                     device=DEV)
    y = ssd_i8.ssd_i8_chunk_scan(
        _dev(case.x), _dev(case.B), _dev(case.C), _dev(case.dt), _dev(case.A), _dev(case.D),
        _dev(case.x_scale), _dev(case.B_scale), _dev(case.C_scale), case.chunk_size,
        init_state=None if h0 is None else _dev(h0), final_state=fs, y_dtype=y_dtype,
        y_scale=y_scale, hadamard=hadamard)
    torch.cuda.synchronize()
    return y.cpu(), fs.cpu().numpy()


@pytest.mark.gpu
@pytest.mark.parametrize("b,L,G,N,Q,init", CASES)
def test_fused_scan_is_exact_on_the_readout_family(_lib, b, L, G, N, Q, init):
    case = W.make_exact_readout(b, L, G, N, Q, seed=L + N)
    h0 = _init_state(case, L) if init else None
    y_ref, fs_ref = oracle.scan(case.x, case.B, case.C, case.dt, case.A, case.D, case.x_scale,
                                case.B_scale, case.C_scale, init_state=h0)[:2]
    # f32 output: bit for bit (every product C_t . B_s read out, the mask, the state path)
    y, fs = _gpu(case, h0, "f32")
    y = y.numpy().astype(np.float64)
    bad = np.argwhere(y != y_ref)
    assert bad.size == 0, f"{len(bad)} outputs differ, first at {bad[0].tolist()}: " \
                          f"{y[tuple(bad[0])]} != {y_ref[tuple(bad[0])]}"
    assert np.array_equal(fs.astype(np.float64), fs_ref)
    # f16 output: the same values (small integers times powers of two are exact in f16)
    y16, _ = _gpu(case, h0, "f16")
    assert np.array_equal(y16.float().numpy().astype(np.float64), y_ref)
    # int8 output with y_scale = scale / 4: codes 4 (C_t . B_s), clamped to +-127 -- exact
    s_y = _scale(case) / 4.0
    q, _ = _gpu(case, h0, "i8", y_scale=s_y)
    q_ref = np.clip(np.rint(y_ref / s_y), -127, 127).astype(np.int8)
    assert np.array_equal(q.numpy(), q_ref)
    # Hadamard-transformed output H y / 8: butterflies of small dyadic values, exact too
    yh, _ = _gpu(case, h0, "f32", hadamard=True)
    assert np.array_equal(yh.numpy().astype(np.float64), oracle.hadamard(y_ref))


# ---------------------------------------------------------------------------------------------
# The same family on the other entry points: packed sequences (the state restarts in each
# sequence, the sequence table, empty and one-token sequences), B and C scales per dstate
# channel (ChunkBMM on f16; power-of-two channel scales keep every operand exact), and the
# fp32-state decode step.
# ---------------------------------------------------------------------------------------------
@pytest.mark.gpu
def test_packed_sequences_are_exact_on_the_readout_family(_lib):
    lengths = [320, 1, 0, 200, 700, 130]
    case, cu = W.make_exact_readout_varlen(lengths, 2, 128, seed=11)
    H, P, N = case.nheads, case.headdim, case.dstate
    nseq = len(lengths)
    T = int(cu[-1])
    fs = torch.full((nseq, H, P, N), float("nan"), dtype=torch.float32, device=DEV)
    y = ssd_i8.ssd_i8_chunk_scan_varlen(
        _dev(case.x[0, :T]), _dev(case.B[0, :T]), _dev(case.C[0, :T]), _dev(case.dt[0, :T]),
        _dev(case.A), _dev(case.D), _dev(case.x_scale), _dev(case.B_scale), _dev(case.C_scale),
        cu, case.chunk_size, final_state=fs, y_dtype="f32")
    torch.cuda.synchronize()
    y = y.cpu().numpy().astype(np.float64)
    fs = fs.cpu().numpy().astype(np.float64)
    for i in range(nseq):
        a, b = int(cu[i]), int(cu[i + 1])
        if b > a:
            yr, fr = oracle.scan(case.x[:, a:b], case.B[:, a:b], case.C[:, a:b], case.dt[:, a:b],
                                 case.A, case.D, case.x_scale, case.B_scale, case.C_scale)[:2]
            assert np.array_equal(y[a:b], yr[0]), f"sequence {i}: y differs"
            assert np.array_equal(fs[i], fr[0]), f"sequence {i}: final state differs"
        else:
            assert np.array_equal(fs[i], np.zeros_like(fs[i])), "empty sequence: state not zero"


@pytest.mark.gpu
@pytest.mark.parametrize("N", [64, 128])
def test_per_channel_scales_are_exact_on_the_readout_family(_lib, N):
    case = W.make_exact_readout(2, 300, 2, N, 256, seed=N)
    rng = np.random.default_rng(N + 1)
    G = case.ngroups
    # s_B[g, n] in {1/4, 1/8}, s_C = 1/2: u = s_B s_C in {1/8, 1/16}, u / max u in {1, 1/2}, so
    # C . (B u / max u) is a multiple of 1/2 below 2^8 in magnitude: exact in f16 and fp32
    case.B_scale = (2.0 ** -rng.integers(2, 4, size=(G, N))).astype(np.float32)
    case.C_scale = np.full((G, N), 0.5, dtype=np.float32)
    y_ref, fs_ref = oracle.scan(case.x, case.B, case.C, case.dt, case.A, case.D, case.x_scale,
                                case.B_scale, case.C_scale)[:2]
    y, fs = _gpu(case, None, "f32")
    assert np.array_equal(y.numpy().astype(np.float64), y_ref)
    assert np.array_equal(fs.astype(np.float64), fs_ref)


@pytest.mark.gpu
@pytest.mark.parametrize("N,hadamard", [(128, False), (16, False), (128, True)])
def test_decode_steps_are_exact_on_the_readout_family(_lib, N, hadamard):
    """Five fp32-state decode steps with A = D = 0, dt and scales powers of two, x, B, C codes
    in {-1, 0, 1} and a state of multiples of 1/8: every update and every y is exact."""
    b, H, P, G = 3, 4, 64, 2
    rng = np.random.default_rng(N + 7)
    state = (rng.integers(-2, 3, size=(b, H, P, N)) / 8.0).astype(np.float32)
    ref = state.astype(np.float64)
    A = np.zeros(H, dtype=np.float32)
    D = np.zeros(H, dtype=np.float32)
    sx = np.full(H, 0.5, dtype=np.float32)
    sb = np.full(G, 0.25, dtype=np.float32)
    sc = np.full(G, 0.5, dtype=np.float32)
    st = _dev(state)
    for step in range(5):
        x = rng.integers(-1, 2, size=(b, H, P)).astype(np.int8)
        B = rng.integers(-1, 2, size=(b, G, N)).astype(np.int8)
        C = rng.integers(-1, 2, size=(b, G, N)).astype(np.int8)
        dt = np.full((b, H), 0.125, dtype=np.float32)
        y_ref = oracle.step(ref, x, B, C, dt, A, D, sx, sb, sc)
        if hadamard:
            y_ref = oracle.hadamard(y_ref)
        y = ssd_i8.ssd_i8_state_update(st, _dev(x), _dev(B), _dev(C), _dev(dt), _dev(A), _dev(D),
                                       _dev(sx), _dev(sb), _dev(sc), y_dtype="f32",
                                       hadamard=hadamard)
        torch.cuda.synchronize()
        assert np.array_equal(y.cpu().numpy().astype(np.float64), y_ref), f"step {step}: y differs"
    assert np.array_equal(st.cpu().numpy().astype(np.float64), ref)


def test_packed_family_matches_the_closed_form_per_sequence():
    """CPU: every token t < L of every packed sequence is carried by exactly one (head, column)
    of each group, and the oracle on each sequence is the closed form of the dense family."""
    lengths = [130, 1, 0, 64, 200]
    case, cu = W.make_exact_readout_varlen(lengths, 2, 32, seed=3)
    P, G = case.headdim, case.ngroups
    per_group = case.nheads // G
    for i, L in enumerate(lengths):
        if L == 0:  # an empty sequence carries no token
            continue
        a = int(cu[i])
        xs = case.x[0, a:a + L]  # [L, H, P]
        for g in range(G):
            ones = xs[:, g * per_group:(g + 1) * per_group].reshape(L, -1).sum(axis=1)
            assert np.array_equal(ones, np.ones(L)), f"sequence {i}, group {g}: one-hot broken"
        sub = W.PrefillCase(
            name="seq", batch=1, seqlen=L, nheads=case.nheads, headdim=P, dstate=case.dstate,
            ngroups=G, chunk_size=case.chunk_size, x=case.x[:, a:a + L], B=case.B[:, a:a + L],
            C=case.C[:, a:a + L], dt=case.dt[:, a:a + L], A=case.A, D=case.D,
            x_scale=case.x_scale, B_scale=case.B_scale, C_scale=case.C_scale)
        y = oracle.scan(sub.x, sub.B, sub.C, sub.dt, sub.A, sub.D, sub.x_scale, sub.B_scale,
                        sub.C_scale)[0]
        assert np.array_equal(y, _closed_form(sub, None)), f"sequence {i}: oracle != closed form"
