"""Pins for the CPU oracle: checks against what the pages and the mathematics fix.

None of these re-types the oracle's loop.  Each compares it with an independent
statement of the same quantity:

* the quadratic (masked "attention") form of the scan -- the state space duality that SSDi8
  builds on (SSDi8 page, Abstract and Figure 1) -- obtained by unrolling the recurrence;
* the A = 0 special case, where the scan is a plain cumulative sum, checked bit-exactly in
  rational arithmetic on dyadic inputs;
* brute force with explicit products of the decay factors in rational arithmetic (L <= 8);
* the error-accumulation identity e_T = sum_t Abar^{T-t} eps_t (Ternary Mamba page, section
  6.2, eq. 2) and its time-varying form;
* continuity: a split prefill handing its state on equals one prefill; a decode step equals
  a length-1 prefill;
* hand-worked fixtures under tests/golden/;
* the ChunkBMM integer matrix against Python integers and numpy's einsum;
* the requantization rule (round half to even, symmetric clamp to +-127).

Planted-mistake tests at the end compile deliberately broken copies of the oracle and check
that these pins reject each of them.
"""
import ctypes
import json
import math
import os
import shutil
import subprocess
import tempfile
from fractions import Fraction

import numpy as np
import pytest

import oracle
from quantized_mamba_ssd_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _case(b=2, L=24, H=4, G=2, P=3, N=5, seed=0, init=True):
    c = W.make_prefill(b, L, H, P, N, G, 8, law="laplace_outliers_all", scales="head", seed=seed,
                       with_init_state=init)
    return c


def _run(c, **kw):
    return oracle.scan(c.x, c.B, c.C, c.dt, c.A, c.D, c.x_scale, c.B_scale, c.C_scale,
                       init_state=c.init_state, **kw)


def _deq(c):
    """Dequantized x [b,l,h,p] and B, C expanded to heads [b,l,h,n]; B/C scales per group [g]
    or per group and dstate channel [g, n]."""
    H, G = c.nheads, c.ngroups
    gi = np.arange(H) // (H // G)
    x = c.x.astype(np.float64) * c.x_scale.astype(np.float64)[None, None, :, None]
    per_group = lambda s: s.astype(np.float64)[None, None, :, None] if s.ndim == 1 else \
        s.astype(np.float64)[None, None, :, :]
    Bf = c.B.astype(np.float64) * per_group(c.B_scale)
    Cf = c.C.astype(np.float64) * per_group(c.C_scale)
    return x, Bf[:, :, gi, :], Cf[:, :, gi, :]


def quadratic_form(c):
    """Unrolled scan: y_t = sum_{s<=t} (prod_{k=s+1..t} a_k) dt_s (C_t . B_s) x_s
    + (prod_{k=0..t} a_k) C_t . h0 + D x_t, with a_k = exp(dt_k A)."""
    x, Bh, Ch = _deq(c)
    bsz, L, H, P = x.shape
    N = Bh.shape[-1]
    dt = c.dt.astype(np.float64)
    y = np.zeros((bsz, L, H, P))
    hL = np.zeros((bsz, H, P, N))
    for b in range(bsz):
        for h in range(H):
            a = np.exp(dt[b, :, h] * np.float64(c.A[h]))
            # decay[t, s] = prod_{k=s+1..t} a_k for s <= t, else 0
            decay = np.zeros((L, L))
            for t in range(L):
                for s in range(t + 1):
                    decay[t, s] = np.prod(a[s + 1:t + 1])
            G_ts = Ch[b, :, h, :] @ Bh[b, :, h, :].T  # C_t . B_s
            M = decay * G_ts * dt[b, :, h][None, :]
            y[b, :, h, :] = M @ x[b, :, h, :] + np.float64(c.D[h]) * x[b, :, h, :]
            h0 = (np.zeros((P, N)) if c.init_state is None
                  else c.init_state[b, h].astype(np.float64))
            for t in range(L):
                y[b, t, h, :] += np.prod(a[:t + 1]) * (h0 @ Ch[b, t, h, :])
            # final state from the same unrolling
            w = np.array([np.prod(a[s + 1:]) * dt[b, s, h] for s in range(L)])
            hL[b, h] = (x[b, :, h, :] * w[:, None]).T @ Bh[b, :, h, :] + np.prod(a) * h0
    return y, hL


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_duality_quadratic_form(seed):
    c = _case(seed=seed)
    y, fs, _ = _run(c)
    yq, hq = quadratic_form(c)
    scale = np.abs(yq).max()
    assert np.abs(y - yq).max() <= 1e-12 * scale
    assert np.abs(fs - hq).max() <= 1e-12 * np.abs(hq).max()


def _dyadic_case(seed, L=16, H=2, G=1, P=3, N=6, A_zero=True):
    rng = np.random.default_rng(seed)
    c = W.make_prefill(1, L, H, P, N, G, 8, law="normal", scales="head", seed=seed)
    c.dt = (2.0 ** -rng.integers(1, 5, size=c.dt.shape)).astype(np.float32)
    c.x_scale = (2.0 ** -rng.integers(1, 4, size=H)).astype(np.float32)
    c.B_scale = (2.0 ** -rng.integers(1, 4, size=G)).astype(np.float32)
    c.C_scale = (2.0 ** -rng.integers(1, 4, size=G)).astype(np.float32)
    c.D = (rng.integers(-8, 9, size=H) / 4.0).astype(np.float32)
    if A_zero:
        c.A = np.zeros(H, dtype=np.float32)
    c.init_state = (rng.integers(-64, 65, size=(1, H, P, N)) / 8.0).astype(np.float32)
    return c


def _exact_cumsum(c):
    """A = 0: h_t = h0 + sum_{s<=t} dt_s x_s B_s^T exactly; y_t = C_t . h_t + D x_t."""
    bsz, L, H, P = c.x.shape
    G, N = c.ngroups, c.dstate
    F = Fraction
    y = np.empty((bsz, L, H, P), dtype=object)
    hL = np.empty((bsz, H, P, N), dtype=object)
    for b in range(bsz):
        for h in range(H):
            g = h // (H // G)
            st = [[F(float(c.init_state[b, h, p, n])) for n in range(N)] for p in range(P)]
            for t in range(L):
                dtv = F(float(c.dt[b, t, h]))
                Bt = [F(float(c.B_scale[g])) * int(c.B[b, t, g, n]) for n in range(N)]
                Ct = [F(float(c.C_scale[g])) * int(c.C[b, t, g, n]) for n in range(N)]
                for p in range(P):
                    xv = F(float(c.x_scale[h])) * int(c.x[b, t, h, p])
                    for n in range(N):
                        st[p][n] += dtv * xv * Bt[n]
                    y[b, t, h, p] = sum(Ct[n] * st[p][n] for n in range(N)) + F(float(c.D[h])) * xv
            for p in range(P):
                for n in range(N):
                    hL[b, h, p, n] = st[p][n]
    return y, hL


@pytest.mark.parametrize("seed", [3, 4])
def test_A_zero_is_exact_cumulative_sum(seed):
    c = _dyadic_case(seed)
    y, fs, _ = _run(c)
    ye, he = _exact_cumsum(c)
    # dyadic inputs make every intermediate exactly representable: bit-exact equality
    assert np.array_equal(y, np.vectorize(float)(ye))
    assert np.array_equal(fs, np.vectorize(float)(he))


def _bruteforce(c):
    """Rational brute force with the decay factors a_k = exp(dt_k A) taken once in fp64:
    h_T = sum_s (prod_{k=s+1..T} a_k) dt_s x_s B_s^T + (prod_{k<=T} a_k) h0."""
    bsz, L, H, P = c.x.shape
    G, N = c.ngroups, c.dstate
    F = Fraction
    y = np.zeros((bsz, L, H, P))
    for b in range(bsz):
        for h in range(H):
            g = h // (H // G)
            a = [F(math.exp(float(c.dt[b, k, h]) * float(c.A[h]))) for k in range(L)]
            dt = [F(float(c.dt[b, k, h])) for k in range(L)]
            xs = [[F(float(c.x_scale[h])) * int(c.x[b, k, h, p]) for p in range(P)] for k in range(L)]
            Bs = [[F(float(c.B_scale[g])) * int(c.B[b, k, g, n]) for n in range(N)] for k in range(L)]
            Cs = [[F(float(c.C_scale[g])) * int(c.C[b, k, g, n]) for n in range(N)] for k in range(L)]
            h0 = [[F(float(c.init_state[b, h, p, n])) for n in range(N)] for p in range(P)]
            for t in range(L):
                for p in range(P):
                    tot = F(0)
                    for n in range(N):
                        hv = h0[p][n]
                        for k in range(t + 1):
                            hv *= a[k]
                        for s in range(t + 1):
                            prod = F(1)
                            for k in range(s + 1, t + 1):
                                prod *= a[k]
                            hv += prod * dt[s] * xs[s][p] * Bs[s][n]
                        tot += Cs[t][n] * hv
                    tot += F(float(c.D[h])) * xs[t][p]
                    y[b, t, h, p] = float(tot)
    return y


def test_bruteforce_rational_L8():
    c = _dyadic_case(7, L=8, H=2, G=1, P=2, N=3, A_zero=False)
    c.A = np.array([-1.25, -7.5], dtype=np.float32)
    y, _, _ = _run(c)
    yb = _bruteforce(c)
    assert np.abs(y - yb).max() <= 1e-14 * np.abs(yb).max()


def test_error_accumulation_constant_decay():
    # constant dt per head => Abar constant; e_T = sum_t Abar^{T-t} eps_t
    c = _case(b=1, L=20, H=2, G=1, P=3, N=4, seed=11, init=False)
    c.dt[:] = c.dt[:, :1, :]
    rng = np.random.default_rng(5)
    eps = rng.standard_normal((1, c.seqlen, c.nheads, c.headdim, c.dstate)) * 1e-3
    _, h_clean, _ = _run(c)
    _, h_pert, _ = _run(c, eps=eps)
    T = c.seqlen
    for h in range(c.nheads):
        abar = math.exp(float(c.dt[0, 0, h]) * float(c.A[h]))
        e_T = sum(abar ** (T - 1 - t) * eps[0, t, h] for t in range(T))
        err = h_pert[0, h] - h_clean[0, h]
        assert np.abs(err - e_T).max() <= 1e-12 * np.abs(e_T).max()


def test_error_accumulation_time_varying():
    c = _case(b=1, L=16, H=3, G=1, P=2, N=3, seed=12, init=True)
    rng = np.random.default_rng(6)
    eps = rng.standard_normal((1, c.seqlen, c.nheads, c.headdim, c.dstate)) * 1e-2
    _, h_clean, _ = _run(c)
    _, h_pert, _ = _run(c, eps=eps)
    T = c.seqlen
    for h in range(c.nheads):
        a = [math.exp(float(c.dt[0, k, h]) * float(c.A[h])) for k in range(T)]
        e_T = sum(np.prod(a[t + 1:]) * eps[0, t, h] for t in range(T))
        err = h_pert[0, h] - h_clean[0, h]
        assert np.abs(err - e_T).max() <= 1e-12 * np.abs(e_T).max()


@pytest.mark.parametrize("split", [1, 7, 13])
def test_split_prefill_hands_state_on(split):
    c = _case(b=2, L=20, H=4, G=2, P=3, N=4, seed=21)
    y, fs, _ = _run(c)
    y1, f1, _ = oracle.scan(c.x[:, :split], c.B[:, :split], c.C[:, :split], c.dt[:, :split], c.A,
                            c.D, c.x_scale, c.B_scale, c.C_scale, init_state=c.init_state)
    y2, f2, _ = oracle.scan(c.x[:, split:], c.B[:, split:], c.C[:, split:], c.dt[:, split:], c.A,
                            c.D, c.x_scale, c.B_scale, c.C_scale, init_state=f1)
    assert np.array_equal(np.concatenate([y1, y2], axis=1), y)
    assert np.array_equal(f2, fs)


def test_decode_step_equals_length_one_prefill():
    d = W.make_decode(3, 2, 4, 5, 6, 2, seed=3)
    st = d.state.astype(np.float64)
    y_step = oracle.step(st, d.x[0], d.B[0], d.C[0], d.dt[0], d.A, d.D, d.x_scale, d.B_scale,
                         d.C_scale)
    y_pf, fs, _ = oracle.scan(d.x[0][:, None], d.B[0][:, None], d.C[0][:, None], d.dt[0][:, None],
                              d.A, d.D, d.x_scale, d.B_scale, d.C_scale, init_state=d.state)
    assert np.array_equal(y_step, y_pf[:, 0])
    assert np.array_equal(st, fs)


def test_zero_B_leaves_skip_term_only():
    c = _case(seed=31, init=False)
    c.B[:] = 0
    y, fs, _ = _run(c)
    x, _, _ = _deq(c)
    assert np.array_equal(y, x * c.D.astype(np.float64)[None, None, :, None])
    assert not fs.any()


def test_zero_dt_keeps_initial_state():
    c = _case(seed=32)
    c.dt[:] = 0
    y, fs, _ = _run(c)
    x, _, Ch = _deq(c)
    expect = np.einsum("bhpn,blhn->blhp", c.init_state.astype(np.float64), Ch) + \
        x * c.D.astype(np.float64)[None, None, :, None]
    assert np.allclose(y, expect, rtol=1e-14, atol=1e-14 * np.abs(expect).max())
    assert np.array_equal(fs, c.init_state.astype(np.float64))


def test_golden_handworked_scan():
    g = json.load(open(os.path.join(GOLDEN, "handworked_scan_L3.json")))
    s = g["shape"]
    shp = (s["batch"], s["seqlen"], s["nheads"], s["headdim"])
    bshp = (s["batch"], s["seqlen"], s["ngroups"], s["dstate"])
    y, fs, _ = oracle.scan(np.array(g["x_q"], np.int8).reshape(shp),
                           np.array(g["B_q"], np.int8).reshape(bshp),
                           np.array(g["C_q"], np.int8).reshape(bshp),
                           np.array(g["dt"], np.float32).reshape(shp[:3]),
                           np.array(g["A"], np.float32), np.array(g["D"], np.float32),
                           np.array(g["x_scale"], np.float32), np.array(g["B_scale"], np.float32),
                           np.array(g["C_scale"], np.float32))
    np.testing.assert_allclose(y.ravel(), g["y"], rtol=g["rtol"])
    np.testing.assert_allclose(fs.ravel(), g["final_state"], rtol=g["rtol"])


def test_golden_handworked_cb():
    g = json.load(open(os.path.join(GOLDEN, "handworked_cb.json")))
    C = np.array(g["C_q"], np.int8).reshape(1, 2, 1, 2)
    B = np.array(g["B_q"], np.int8).reshape(1, 2, 1, 2)
    cb = oracle.chunk_cb(C, B, 2)
    assert cb[0, 0, 0].tolist() == g["CB"]


def test_chunk_cb_against_python_integers_and_einsum():
    rng = np.random.default_rng(8)
    bsz, L, G, N, Q = 2, 10, 2, 5, 4
    C = rng.integers(-127, 128, size=(bsz, L, G, N), dtype=np.int8)
    B = rng.integers(-127, 128, size=(bsz, L, G, N), dtype=np.int8)
    cb = oracle.chunk_cb(C, B, Q)
    nch = (L + Q - 1) // Q
    assert cb.shape == (bsz, nch, G, Q, Q)
    for b in range(bsz):
        for c in range(nch):
            for g in range(G):
                for t in range(Q):
                    for s in range(Q):
                        lt, ls = c * Q + t, c * Q + s
                        ref = 0
                        if lt < L and ls < L:
                            ref = sum(int(C[b, lt, g, n]) * int(B[b, ls, g, n]) for n in range(N))
                        assert cb[b, c, g, t, s] == ref
    # a full-size group block against numpy's integer einsum
    C2 = rng.integers(-127, 128, size=(1, 256, 1, 128), dtype=np.int8)
    B2 = rng.integers(-127, 128, size=(1, 256, 1, 128), dtype=np.int8)
    ref = np.einsum("tn,sn->ts", C2[0, :, 0].astype(np.int64), B2[0, :, 0].astype(np.int64))
    assert np.array_equal(oracle.chunk_cb(C2, B2, 256)[0, 0, 0], ref)


def test_requant_rule():
    y = np.array([0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 126.5, 127.49, 300.0, -127.5, -1e9, 0.49999])
    q = oracle.requant(y, 1.0)
    assert q.tolist() == [0, 2, 2, 0, -2, -2, 126, 127, 127, -127, -127, 0]
    q = oracle.requant(np.array([0.3, -0.3, 0.05]), 0.1)
    assert q.tolist() == [3, -3, 0]  # 0.05/0.1 = 0.5 -> ties to even (0)


# ----------------------------------------------------------------------------------------
# B and C scales per dstate channel (the per-N axis of SSDi8's quantization-axis table)
# ----------------------------------------------------------------------------------------
def _per_n_case(seed=7, b=1, L=20, H=4, G=2, P=3, N=6):
    c = _case(b=b, L=L, H=H, G=G, P=P, N=N, seed=seed)
    rng = np.random.default_rng(seed + 100)
    c.B_scale = (c.B_scale[:, None] * rng.uniform(0.25, 4.0, size=(G, N))).astype(np.float32)
    c.C_scale = (c.C_scale[:, None] * rng.uniform(0.25, 4.0, size=(G, N))).astype(np.float32)
    return c


def test_per_n_scales_constant_over_n_equal_per_group():
    c = _case(seed=5)
    y, fs, _ = _run(c)
    N = c.dstate
    c.B_scale = np.repeat(c.B_scale[:, None], N, axis=1)
    c.C_scale = np.repeat(c.C_scale[:, None], N, axis=1)
    y2, fs2, _ = _run(c)
    assert np.array_equal(y, y2) and np.array_equal(fs, fs2)


@pytest.mark.parametrize("seed", [7, 8])
def test_per_n_duality_quadratic_form(seed):
    c = _per_n_case(seed=seed)
    y, fs, _ = _run(c)
    yq, hq = quadratic_form(c)
    assert np.abs(y - yq).max() <= 1e-12 * np.abs(yq).max()
    assert np.abs(fs - hq).max() <= 1e-12 * np.abs(hq).max()


def test_per_n_scale_acts_on_its_own_channel():
    # h_t[p, n] is linear in s_B[g, n] alone and does not involve C: doubling s_B[g, k] (a
    # power of two, so exactly) doubles column k of the states of group g's heads and nothing
    # else; doubling s_C[g, k] leaves every state as it was and changes y
    c = _per_n_case(seed=9)
    c.init_state = None
    y, fs, _ = _run(c)
    H, G = c.nheads, c.ngroups
    g, k = 1, 4
    heads = np.arange(H)[np.arange(H) // (H // G) == g]
    c2 = _per_n_case(seed=9)
    c2.init_state = None
    c2.B_scale = c2.B_scale.copy()
    c2.B_scale[g, k] *= 2
    y2, fs2, _ = _run(c2)
    expect = fs.copy()
    expect[:, heads, :, k] *= 2
    assert np.array_equal(fs2, expect)
    c3 = _per_n_case(seed=9)
    c3.init_state = None
    c3.C_scale = c3.C_scale.copy()
    c3.C_scale[g, k] *= 2
    y3, fs3, _ = _run(c3)
    assert np.array_equal(fs3, fs)
    assert not np.array_equal(y3[:, :, heads], y[:, :, heads])
    others = np.setdiff1d(np.arange(H), heads)
    assert np.array_equal(y3[:, :, others], y[:, :, others])


# ----------------------------------------------------------------------------------------
# planted mistakes: each broken copy of the oracle must fail at least one pin above
# ----------------------------------------------------------------------------------------
MUTANTS = {
    "drop_skip_term": ("j->y[(bt * H + h) * P + p] = acc + (double)j->D[h] * xv;",
                       "j->y[(bt * H + h) * P + p] = acc;"),
    "flip_decay_sign": ("exp(dtv * (double)j->A[h])", "exp(-dtv * (double)j->A[h])"),
    "drop_dt_on_input": ("row[n] = abar * row[n] + dtv * xv * Bt[n];",
                         "row[n] = abar * row[n] + xv * Bt[n];"),
    "C_reads_B": ("Ct[n] = sc * (double)j->C[", "Ct[n] = sc * (double)j->B["),
    "per_n_scale_of_first_channel": ("j->sB[g * N + n] : j->sB[g]", "j->sB[g * N] : j->sB[g]"),
    "per_n_B_scale_read_from_C": ("(double)(j->bc_per_n ? j->sB[g * N + n]",
                                  "(double)(j->bc_per_n ? j->sC[g * N + n]"),
    "wrong_group_index": ("const int g = h / (H / G);", "const int g = h % G;"),
    "cb_transposed": ("(int64_t)C[(((size_t)b * L + lt) * G + g) * N + n] *\n                                       (int64_t)B[(((size_t)b * L + ls) * G + g) * N + n]",
                      "(int64_t)C[(((size_t)b * L + ls) * G + g) * N + n] *\n                                       (int64_t)B[(((size_t)b * L + lt) * G + g) * N + n]"),
    "requant_truncates": ("double r = nearbyint(y[i] / y_scale);", "double r = trunc(y[i] / y_scale);"),
}


def _pins_pass():
    checks = [
        lambda: test_duality_quadratic_form(0),
        lambda: test_A_zero_is_exact_cumulative_sum(3),
        test_error_accumulation_time_varying,
        test_golden_handworked_scan,
        test_golden_handworked_cb,
        test_chunk_cb_against_python_integers_and_einsum,
        test_requant_rule,
        test_zero_B_leaves_skip_term_only,
        test_per_n_scales_constant_over_n_equal_per_group,
        lambda: test_per_n_duality_quadratic_form(7),
        test_per_n_scale_acts_on_its_own_channel,
    ]
    for chk in checks:
        try:
            chk()
        except AssertionError:
            return False
    return True


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_pins_reject_planted_mistake(mutant, monkeypatch):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "ssd_oracle.c")).read()
    old, new = MUTANTS[mutant]
    assert src.count(old) == 1, f"mutation site for {mutant} not found"
    tmp = tempfile.mkdtemp(prefix="oracle_mutant_")
    try:
        path = os.path.join(tmp, "m.c")
        with open(path, "w") as f:
            f.write(src.replace(old, new))
        so = os.path.join(tmp, "libm.so")
        subprocess.run(["gcc", "-O2", "-std=c11", "-D_GNU_SOURCE", "-ffp-contract=off", "-fPIC",
                        "-shared", "-o", so, path, "-lm", "-lpthread"], check=True)
        good = oracle.load()
        lib = ctypes.CDLL(so)
        for name in ("ssd_oracle_scan", "ssd_oracle_scan_pern", "ssd_oracle_step",
                     "ssd_oracle_chunk_cb", "ssd_oracle_requant"):
            getattr(lib, name).restype = getattr(good, name).restype
            getattr(lib, name).argtypes = getattr(good, name).argtypes
        monkeypatch.setattr(oracle, "_lib", lib)
        assert not _pins_pass(), f"planted mistake {mutant} passed every pin"
    finally:
        shutil.rmtree(tmp, ignore_errors=True)


# ---- int8 cached decode state (quantize_state / step_q8) ----

def _random_state(seed, shape=(2, 3, 8, 16), sd=0.7):
    return np.random.default_rng(seed).normal(0.0, sd, size=shape)


def test_quantize_state_rule():
    st = _random_state(21)
    codes, scales = oracle.quantize_state(st)
    deq = codes.astype(np.float64) * scales[:, :, None, None]
    # every element within half a step of its code, the largest one at the end of the range
    assert (np.abs(deq - st) <= 0.5 * scales[:, :, None, None] * (1 + 1e-12)).all()
    for b in range(st.shape[0]):
        for h in range(st.shape[1]):
            i = np.unravel_index(np.abs(st[b, h]).argmax(), st[b, h].shape)
            assert abs(int(codes[b, h][i])) == 127
            assert np.isclose(scales[b, h], np.abs(st[b, h]).max() / 127.0, rtol=0, atol=0)
    # an all-zero state quantizes to scale 0 and codes 0
    z_codes, z_scales = oracle.quantize_state(np.zeros((1, 2, 4, 16)))
    assert (z_codes == 0).all() and (z_scales == 0).all()


def test_quantize_state_is_idempotent_on_codes():
    st = _random_state(22)
    codes, scales = oracle.quantize_state(st)
    codes2, scales2 = oracle.quantize_state(codes.astype(np.float64) * scales[:, :, None, None])
    assert np.array_equal(codes, codes2)
    assert np.allclose(scales, scales2, rtol=1e-15, atol=0)


def test_step_q8_with_zero_dt_keeps_the_cache():
    # dt = 0: decay exp(0) = 1 and no input, so the dequantised state comes back unchanged
    bsz, H, P, N, G = 2, 4, 8, 16, 2
    codes, scales = oracle.quantize_state(_random_state(23, (bsz, H, P, N)))
    rng = np.random.default_rng(24)
    x = rng.integers(-127, 128, size=(bsz, H, P), dtype=np.int8)
    B = rng.integers(-127, 128, size=(bsz, G, N), dtype=np.int8)
    C = rng.integers(-127, 128, size=(bsz, G, N), dtype=np.int8)
    A = -np.exp(rng.uniform(0, np.log(16), H)).astype(np.float32)
    D = rng.normal(size=H).astype(np.float32)
    sx = np.full(H, 0.02, np.float32)
    sB = np.full(G, 0.03, np.float32)
    sC = np.full(G, 0.04, np.float32)
    dt = np.zeros((bsz, H), np.float32)
    y, c2, s2 = oracle.step_q8(codes, scales, x, B, C, dt, A, D, sx, sB, sC)
    assert np.array_equal(codes, c2)
    assert np.allclose(scales, s2, rtol=1e-15, atol=0)
    # y = C h + D x of the unchanged state
    h = codes.astype(np.float64) * scales[:, :, None, None]
    g = np.arange(H) // (H // G)
    yref = np.einsum("bhpn,bhn->bhp", h, C[:, g].astype(np.float64) * sC[g][None, :, None]) \
        + D.astype(np.float64)[None, :, None] * sx.astype(np.float64)[None, :, None] * x
    assert np.allclose(y, yref, rtol=1e-12, atol=1e-12)


def _golden_step_q8_inputs():
    with open(os.path.join(GOLDEN, "handworked_step_q8.json")) as f:
        g = json.load(f)
    codes = np.array(g["codes"], np.int8)[None, None]
    scale = np.array([[g["scale"]]], np.float64)
    ins = dict(x=np.array(g["x_q"], np.int8)[None, None], B=np.array(g["B_q"], np.int8)[None, None],
               C=np.array(g["C_q"], np.int8)[None, None], dt=np.array([g["dt"]], np.float32),
               A=np.array(g["A"], np.float32), D=np.array(g["D"], np.float32),
               x_scale=np.array(g["x_scale"], np.float32),
               B_scale=np.array(g["B_scale"], np.float32),
               C_scale=np.array(g["C_scale"], np.float32))
    return g, codes, scale, ins


def test_golden_handworked_step_q8():
    # a step whose max |h| grows: the fresh scale differs from the incoming one
    g, codes, scale, ins = _golden_step_q8_inputs()
    y, c2, s2 = oracle.step_q8(codes, scale, **ins)
    assert np.allclose(y[0, 0], g["y"], rtol=g["rtol"], atol=0)
    assert np.array_equal(c2[0, 0], np.array(g["new_codes"], np.int8))
    assert np.isclose(s2[0, 0], g["new_scale"], rtol=g["rtol"], atol=0)
    assert not np.isclose(s2[0, 0], g["scale"], rtol=1e-2)


def test_step_q8_codes_follow_the_fresh_scale():
    # random caches and inputs: each new code is within half a fresh step of the fp64 step of
    # the dequantised cache, the largest element gets code +-127 and the scale is its |h| / 127
    bsz, H, P, N, G = 2, 4, 8, 16, 2
    codes, scales = oracle.quantize_state(_random_state(25, (bsz, H, P, N), sd=0.3))
    rng = np.random.default_rng(26)
    x = rng.integers(-127, 128, size=(bsz, H, P), dtype=np.int8)
    B = rng.integers(-127, 128, size=(bsz, G, N), dtype=np.int8)
    C = rng.integers(-127, 128, size=(bsz, G, N), dtype=np.int8)
    A = -np.exp(rng.uniform(0, np.log(16), H)).astype(np.float32)
    D = rng.normal(size=H).astype(np.float32)
    sx, sB, sC = (np.full(k, v, np.float32) for k, v in ((H, 0.02), (G, 0.03), (G, 0.04)))
    dt = rng.uniform(0.05, 0.3, size=(bsz, H)).astype(np.float32)
    y, c2, s2 = oracle.step_q8(codes, scales, x, B, C, dt, A, D, sx, sB, sC)
    h = np.ascontiguousarray(codes.astype(np.float64) * scales[:, :, None, None])
    yref = oracle.step(h, x, B, C, dt, A, D, sx, sB, sC)
    assert np.array_equal(y, yref)
    m = np.abs(h).reshape(bsz, H, -1).max(axis=2)
    assert np.allclose(s2, m / 127.0, rtol=1e-15, atol=0)
    assert (np.abs(c2.astype(np.float64) * s2[:, :, None, None] - h)
            <= 0.5 * s2[:, :, None, None] * (1 + 1e-12)).all()
    assert (np.abs(c2).reshape(bsz, H, -1).max(axis=2) == 127).all()


def _step_q8_with_incoming_scale(codes, scales, x, B, C, dt, A, D, x_scale, B_scale, C_scale):
    # planted mistake: requantise the updated state with the scale the cache came in with
    state = np.ascontiguousarray(codes.astype(np.float64) * scales[:, :, None, None])
    y = oracle.step(state, x, B, C, dt, A, D, x_scale, B_scale, C_scale)
    c2 = np.zeros_like(codes)
    for b in range(codes.shape[0]):
        for h in range(codes.shape[1]):
            if scales[b, h] > 0:
                c2[b, h] = oracle.requant(state[b, h], scales[b, h])
    return y, c2, np.array(scales, dtype=np.float64)


def _step_q8_keeping_codes(codes, scales, x, B, C, dt, A, D, x_scale, B_scale, C_scale):
    # planted mistake: return the incoming codes and scale
    state = np.ascontiguousarray(codes.astype(np.float64) * scales[:, :, None, None])
    y = oracle.step(state, x, B, C, dt, A, D, x_scale, B_scale, C_scale)
    return y, codes.copy(), np.array(scales, dtype=np.float64)


@pytest.mark.parametrize("broken", [_step_q8_with_incoming_scale, _step_q8_keeping_codes])
def test_step_q8_pins_reject_planted_mistake(broken, monkeypatch):
    monkeypatch.setattr(oracle, "step_q8", broken)
    failed = 0
    for chk in (test_golden_handworked_step_q8, test_step_q8_with_zero_dt_keeps_the_cache,
                test_step_q8_codes_follow_the_fresh_scale):
        try:
            chk()
        except AssertionError:
            failed += 1
    assert failed > 0, f"planted mistake {broken.__name__} passed every step_q8 pin"


# ---- Hadamard output transform ----

def test_hadamard_is_an_involution():
    y = np.random.default_rng(31).normal(size=(5, 3, 64))
    assert np.allclose(oracle.hadamard(oracle.hadamard(y)), y, rtol=0, atol=1e-12)


def test_hadamard_of_constant_and_one_hot_rows():
    P = 64
    c = np.full(P, 0.5)
    out = oracle.hadamard(c)
    assert np.isclose(out[0], 0.5 * np.sqrt(P)) and np.allclose(out[1:], 0.0, atol=1e-15)
    for p in (0, 1, 5, 63):
        e = np.zeros(P)
        e[p] = 1.0
        col = oracle.hadamard(e)
        # Sylvester order: entry q is (-1)^popcount(p & q) / sqrt(P)
        want = np.array([(-1) ** bin(p & q).count("1") for q in range(P)]) / np.sqrt(P)
        assert np.allclose(col, want, rtol=0, atol=1e-15)
