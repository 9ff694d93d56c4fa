"""Pins for the float64 oracle: facts fixed by the pages and by plain mathematics.

Every pin takes an oracle object (``.scan`` / ``.step``) and raises AssertionError
when the oracle disagrees. The test suite runs them against the oracle as built,
and against deliberately broken copies of its source (tests/test_oracle_mutants.py)
to show that each plausible mistake fails at least one pin.

None of these pins re-types the oracle's loop. Each one computes the expected
value by a different route: a convolution, a closed form, an unrolled sum, a
chunked evaluation with the associative combine, or a limit.
"""
import math

import numpy as np

DT_F32 = "f32"


def _rng(seed):
    return np.random.default_rng(seed)


def _rel(err, ref):
    ref = np.max(np.abs(ref))
    return float(np.max(np.abs(err)) / (ref if ref > 0 else 1.0))


def _softplus(v):
    # log(1 + e^v) through logaddexp: a different evaluation from the oracle's log1p form.
    return np.logaddexp(0.0, v)


def _sigma(v):
    return 1.0 / (1.0 + np.exp(-v))


def _bf16_bits(a):
    """float32 -> bfloat16 bit patterns, round to nearest even (test-side helper)."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)
    return r


def _bf16_value(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def pin_lti_convolution(orc, dtype=DT_F32, seed=1):
    """Time-invariant case equals a convolution with K_k = sum_n C_n Abar_n^k Bbar_n.

    [SSM encyclopaedia (urworte.de), "Methodische Grundlagen": convolution form for
    training, recurrence for inference]; [SSM blog (shakilmahmud.com), section 3, dual
    form]; [Mamba summary (azimuth.plus), LTI paragraph: constant parameters give the
    convolution shortcut]. Constant Delta (dt_raw = 0), B and C constant over time,
    no gate; A has distinct entries per (d, n) so that a swapped index shows.
    """
    rng = _rng(seed)
    Bsz, L, Dm, N = 2, 48, 3, 5
    bias = np.array([-2.0, -0.3, 0.7], dtype=np.float32)
    A = (-(0.4 + np.arange(N)[None, :] + 0.37 * np.arange(Dm)[:, None])).astype(np.float32)
    beta = rng.standard_normal((Bsz, N)).astype(np.float32)
    gamma = rng.standard_normal((Bsz, N)).astype(np.float32)
    Dskip = rng.standard_normal(Dm).astype(np.float32)
    x32 = rng.standard_normal((Bsz, L, Dm)).astype(np.float32)
    Bm32 = np.repeat(beta[:, None, :], L, axis=1)
    Cm32 = np.repeat(gamma[:, None, :], L, axis=1)
    if dtype == "bf16":
        x, Bm, Cm = _bf16_bits(x32), _bf16_bits(Bm32), _bf16_bits(Cm32)
        xv, bv, gv = _bf16_value(x), _bf16_value(Bm)[:, 0, :], _bf16_value(Cm)[:, 0, :]
        dt = np.zeros((Bsz, L, Dm), dtype=np.uint16)
    else:
        x, Bm, Cm = x32, Bm32, Cm32
        xv, bv, gv = x32.astype(np.float64), beta.astype(np.float64), gamma.astype(np.float64)
        dt = np.zeros((Bsz, L, Dm), dtype=np.float32)
    y, _ = orc.scan(x, dt, A, Bm, Cm, D=Dskip, dt_bias=bias, dtype=dtype)
    delta = _softplus(bias.astype(np.float64))
    expect = np.zeros((Bsz, L, Dm))
    for b in range(Bsz):
        for d in range(Dm):
            abar = np.exp(delta[d] * A[d].astype(np.float64))
            k = np.arange(L)
            K = (gv[b][None, :] * np.power(abar[None, :], k[:, None]) * delta[d] * bv[b][None, :]).sum(1)
            for t in range(L):
                expect[b, t, d] = np.dot(K[: t + 1], xv[b, t::-1, d]) + Dskip[d] * xv[b, t, d]
    e = _rel(y - expect, expect)
    assert e < 1e-12, f"LTI convolution mismatch: rel err {e:.3e}"


def pin_theorem1_closed_form(orc, seed=2):
    """State size 1, A = -1: Abar = exp(-softplus(u)) = 1 - sigma(u), so with Bbar = Delta B
    h_L = sum_t prod_{s>t} (1 - sigma(u_s)) * softplus(u_t) * B_t * x_t (h0 = 0).

    [Mamba summary (azimuth.plus), Theorem 1 paragraph: N = 1 selective SSM is a gated RNN].
    """
    rng = _rng(seed)
    Bsz, L, Dm = 2, 40, 3
    x = rng.standard_normal((Bsz, L, Dm)).astype(np.float32)
    dt = (0.8 * rng.standard_normal((Bsz, L, Dm))).astype(np.float32)
    Bm = rng.standard_normal((Bsz, L, 1)).astype(np.float32)
    Cm = rng.standard_normal((Bsz, L, 1)).astype(np.float32)
    bias = np.array([-1.0, 0.0, 0.5], dtype=np.float32)
    A = -np.ones((Dm, 1), dtype=np.float32)
    _, h = orc.scan(x, dt, A, Bm, Cm, dt_bias=bias)
    u = dt.astype(np.float64) + bias[None, None, :]
    keep = 1.0 - _sigma(u)                       # the gate's "keep" factor
    inject = _softplus(u) * Bm.astype(np.float64) * x
    expect = np.zeros((Bsz, Dm))
    for t in range(L):
        expect += np.prod(keep[:, t + 1:, :], axis=1) * inject[:, t, :]
    e = _rel(h[:, :, 0] - expect, expect)
    assert e < 1e-12, f"Theorem 1 closed form mismatch: rel err {e:.3e}"


def pin_theorem1_gated_rnn(orc, seed=3):
    """With the exact zero-order hold, N = 1, A = -1, B = C = 1, D = 0 and no gate the
    scan is exactly the gated RNN h_t = (1 - g_t) h_{t-1} + g_t x_t, g_t = sigma(u_t),
    and y_t = h_t. [Mamba summary (azimuth.plus), Theorem 1 paragraph]."""
    rng = _rng(seed)
    Bsz, L, Dm = 1, 64, 4
    x = rng.standard_normal((Bsz, L, Dm)).astype(np.float32)
    dt = rng.standard_normal((Bsz, L, Dm)).astype(np.float32)
    h0 = rng.standard_normal((Bsz, Dm, 1)).astype(np.float32)
    ones = np.ones((Bsz, L, 1), dtype=np.float32)
    A = -np.ones((Dm, 1), dtype=np.float32)
    y, h = orc.scan(x, dt, A, ones, ones, h0=h0, exact_zoh=True)
    g = _sigma(dt.astype(np.float64))
    hh = h0[:, :, 0].astype(np.float64)
    expect = np.zeros((Bsz, L, Dm))
    for t in range(L):
        hh = (1.0 - g[:, t, :]) * hh + g[:, t, :] * x[:, t, :]
        expect[:, t, :] = hh
    e = _rel(y - expect, expect)
    assert e < 1e-12, f"gated-RNN form mismatch: rel err {e:.3e}"
    assert _rel(h[:, :, 0] - hh, hh) < 1e-12


def pin_small_delta_keeps_state(orc, seed=4):
    """Delta -> 0 (dt_bias = -40): the state is kept and the input ignored, so
    h_L = h0 and y_t = (C_t . h0 + D x_t) silu(z_t).
    [Mamba summary (azimuth.plus), selectivity paragraph: small Delta keeps the state]."""
    rng = _rng(seed)
    Bsz, L, Dm, N = 2, 30, 3, 4
    x = rng.standard_normal((Bsz, L, Dm)).astype(np.float32)
    dt = (0.5 * rng.standard_normal((Bsz, L, Dm))).astype(np.float32)
    z = rng.standard_normal((Bsz, L, Dm)).astype(np.float32)
    Bm = rng.standard_normal((Bsz, L, N)).astype(np.float32)
    Cm = rng.standard_normal((Bsz, L, N)).astype(np.float32)
    A = -np.tile(np.arange(1, N + 1, dtype=np.float32), (Dm, 1))
    Dskip = rng.standard_normal(Dm).astype(np.float32)
    h0 = rng.standard_normal((Bsz, Dm, N)).astype(np.float32)
    bias = np.full(Dm, -40.0, dtype=np.float32)
    y, h = orc.scan(x, dt, A, Bm, Cm, D=Dskip, z=z, dt_bias=bias, h0=h0)
    assert _rel(h - h0, h0) < 1e-15, "small Delta must keep the state"
    zz = z.astype(np.float64)
    expect = (np.einsum("bln,bdn->bld", Cm.astype(np.float64), h0.astype(np.float64))
              + Dskip.astype(np.float64)[None, None, :] * x) * zz * _sigma(zz)
    e = _rel(y - expect, expect)
    assert e < 1e-14, f"small-Delta readout mismatch: rel err {e:.3e}"


def pin_large_delta_resets_state(orc, seed=5):
    """Large Delta (dt_bias = +50, A <= -1): Abar <= e^-50, the state is reset onto the
    current input. With Bbar = Delta B: h_t = Delta_t B_t x_t; with the exact ZOH:
    h_t = -B_t x_t / A. [Mamba summary (azimuth.plus), selectivity paragraph: large Delta
    resets the state and absorbs the new input]."""
    rng = _rng(seed)
    Bsz, L, Dm, N = 2, 25, 3, 4
    x = rng.standard_normal((Bsz, L, Dm)).astype(np.float32)
    dt = (0.5 * rng.standard_normal((Bsz, L, Dm))).astype(np.float32)
    Bm = rng.standard_normal((Bsz, L, N)).astype(np.float32)
    Cm = rng.standard_normal((Bsz, L, N)).astype(np.float32)
    A = -np.tile(np.arange(1, N + 1, dtype=np.float32), (Dm, 1))
    Dskip = rng.standard_normal(Dm).astype(np.float32)
    h0 = rng.standard_normal((Bsz, Dm, N)).astype(np.float32)
    bias = np.full(Dm, 50.0, dtype=np.float32)
    delta = _softplus(dt.astype(np.float64) + 50.0)
    y, h = orc.scan(x, dt, A, Bm, Cm, D=Dskip, dt_bias=bias, h0=h0)
    hL = delta[:, -1, :, None] * Bm[:, -1, None, :] * x[:, -1, :, None]
    assert _rel(h - hL, hL) < 1e-14, "large Delta must reset the state onto the input"
    expect = (np.einsum("bln,bld->bld", Cm.astype(np.float64) * Bm, delta * x)
              + Dskip.astype(np.float64) * x)
    assert _rel(y - expect, expect) < 1e-14
    # Exact zero-order hold: the reset state is -B x / A.
    y2, h2 = orc.scan(x, dt, A, Bm, Cm, D=None, dt_bias=bias, h0=h0, exact_zoh=True)
    hL2 = -Bm[:, -1, None, :].astype(np.float64) * x[:, -1, :, None] / A[None].astype(np.float64)
    assert _rel(h2 - hL2, hL2) < 1e-14, "exact ZOH reset state must be -B x / A"


def _brute(x, dt, A, Bm, Cm, Dskip, z, bias, h0, softplus=True, exact_zoh=False):
    """h_t = (prod_{r<=t} Abar_r) h0 + sum_{s<=t} (prod_{s<r<=t} Abar_r) Bbar_s x_s,
    written out term by term (tiny sizes only)."""
    Bsz, L, Dm = x.shape
    N = A.shape[1]
    y = np.zeros((Bsz, L, Dm))
    hL = np.zeros((Bsz, Dm, N))
    for b in range(Bsz):
        for d in range(Dm):
            u = [float(dt[b, t, d]) + float(bias[d]) for t in range(L)]
            delta = [math.log1p(math.exp(v)) if (softplus and v < 30) else v for v in u]
            for t in range(L):
                yt = 0.0
                for n in range(N):
                    a = float(A[d, n])
                    abar = [math.exp(delta[r] * a) for r in range(L)]
                    hn = math.prod(abar[: t + 1]) * float(h0[b, d, n])
                    for s in range(t + 1):
                        if exact_zoh:
                            bbar = (math.expm1(delta[s] * a) / a) * float(Bm[b, s, n])
                        else:
                            bbar = delta[s] * float(Bm[b, s, n])
                        hn += math.prod(abar[s + 1: t + 1]) * bbar * float(x[b, s, d])
                    yt += float(Cm[b, t, n]) * hn
                    if t == L - 1:
                        hL[b, d, n] = hn
                yt += float(Dskip[d]) * float(x[b, t, d])
                if z is not None:
                    zv = float(z[b, t, d])
                    yt *= zv / (1.0 + math.exp(-zv))
                y[b, t, d] = yt
    return y, hL


def pin_bruteforce(orc, seed=6):
    """Tiny random cases against the unrolled sum (all flags, both dtypes).
    [Mamba summary (azimuth.plus), hardware-aware algorithm paragraph: the recurrence
    h_t = Abar_t h_{t-1} + Bbar_t x_t; block paragraph: SiLU gate]."""
    rng = _rng(seed)
    for case, (Bsz, L, Dm, N, dtype, softplus, ezoh, gate) in enumerate([
            (2, 9, 3, 4, "f32", True, False, True),
            (1, 12, 2, 3, "bf16", True, False, True),
            (2, 7, 3, 2, "f32", False, False, False),
            (1, 10, 3, 4, "f32", True, True, True),
            (1, 1, 5, 4, "bf16", True, False, True)]):
        x32 = rng.standard_normal((Bsz, L, Dm)).astype(np.float32)
        dt32 = (0.7 * rng.standard_normal((Bsz, L, Dm))).astype(np.float32)
        if not softplus:
            dt32 = np.abs(dt32)
        z32 = rng.standard_normal((Bsz, L, Dm)).astype(np.float32)
        B32 = rng.standard_normal((Bsz, L, N)).astype(np.float32)
        C32 = rng.standard_normal((Bsz, L, N)).astype(np.float32)
        A = (-rng.uniform(0.2, 3.0, (Dm, N))).astype(np.float32)
        Dskip = rng.standard_normal(Dm).astype(np.float32)
        bias = rng.uniform(-2.0, 0.5, Dm).astype(np.float32)
        if not softplus:
            bias = np.abs(bias)
        h0 = rng.standard_normal((Bsz, Dm, N)).astype(np.float32)
        if dtype == "bf16":
            x, dt, z, Bm, Cm = (_bf16_bits(a) for a in (x32, dt32, z32, B32, C32))
            xv, dtv, zv, Bv, Cv = (_bf16_value(a) for a in (x, dt, z, Bm, Cm))
        else:
            x, dt, z, Bm, Cm = x32, dt32, z32, B32, C32
            xv, dtv, zv, Bv, Cv = x32, dt32, z32, B32, C32
        y, h = orc.scan(x, dt, A, Bm, Cm, D=Dskip, z=z if gate else None, dt_bias=bias, h0=h0,
                        dtype=dtype, delta_softplus=softplus, exact_zoh=ezoh)
        ye, he = _brute(xv, dtv, A, Bv, Cv, Dskip, zv if gate else None, bias, h0, softplus, ezoh)
        assert _rel(y - ye, ye) < 1e-13, f"brute-force case {case}: y mismatch {_rel(y - ye, ye):.3e}"
        assert _rel(h - he, he) < 1e-13, f"brute-force case {case}: h mismatch"


def chunked_scan(delta, x, A, Bm, Cm, Dskip, z, h0, chunk):
    """The same scan evaluated chunk by chunk with the associative combine
    (a1, b1) o (a2, b2) = (a1 a2, a2 b1 + b2): per chunk the aggregate (P, S) from a
    zero state, carried across chunks, then h_t = cumprod_t * H_in + local_t inside.
    Inputs are float64 arrays for one (b, d) row. [Mamba summary (azimuth.plus),
    hardware-aware algorithm paragraph: the recurrence is associative, so a
    parallel prefix scan applies]."""
    L = x.shape[0]
    N = A.shape[0]
    H = h0.copy()
    y = np.zeros(L)
    for c0 in range(0, L, chunk):
        c1 = min(L, c0 + chunk)
        abar = np.exp(delta[c0:c1, None] * A[None, :])
        bx = delta[c0:c1, None] * Bm[c0:c1] * x[c0:c1, None]
        P = np.ones(N)
        S = np.zeros(N)
        cum = np.zeros((c1 - c0, N))
        loc = np.zeros((c1 - c0, N))
        for i in range(c1 - c0):            # local prefix from a zero state
            P, S = P * abar[i], abar[i] * S + bx[i]
            cum[i], loc[i] = P, S
        h = cum * H[None, :] + loc           # apply the incoming carry
        y[c0:c1] = (Cm[c0:c1] * h).sum(1) + Dskip * x[c0:c1]
        H = P * H + S                        # carry for the next chunk
    if z is not None:
        y = y * z * _sigma(z)
    return y, H


def pin_associative_chunks(orc, seed=7):
    """The chunked evaluation (chunk sizes 1, 7, 64) equals the sequential oracle."""
    rng = _rng(seed)
    Bsz, L, Dm, N = 1, 150, 2, 4
    x = rng.standard_normal((Bsz, L, Dm)).astype(np.float32)
    dt = (0.5 * rng.standard_normal((Bsz, L, Dm))).astype(np.float32)
    z = rng.standard_normal((Bsz, L, Dm)).astype(np.float32)
    Bm = rng.standard_normal((Bsz, L, N)).astype(np.float32)
    Cm = rng.standard_normal((Bsz, L, N)).astype(np.float32)
    A = (-rng.uniform(0.5, 4.0, (Dm, N))).astype(np.float32)
    Dskip = rng.standard_normal(Dm).astype(np.float32)
    bias = np.array([-3.0, -1.0], dtype=np.float32)
    h0 = rng.standard_normal((Bsz, Dm, N)).astype(np.float32)
    y, h = orc.scan(x, dt, A, Bm, Cm, D=Dskip, z=z, dt_bias=bias, h0=h0)
    for chunk in (1, 7, 64):
        for d in range(Dm):
            delta = _softplus(dt[0, :, d].astype(np.float64) + bias[d])
            yc, Hc = chunked_scan(delta, x[0, :, d].astype(np.float64), A[d].astype(np.float64),
                                  Bm[0].astype(np.float64), Cm[0].astype(np.float64),
                                  float(Dskip[d]), z[0, :, d].astype(np.float64),
                                  h0[0, d].astype(np.float64), chunk)
            assert _rel(y[0, :, d] - yc, yc) < 1e-12, f"chunk {chunk}: y mismatch"
            assert _rel(h[0, d] - Hc, Hc) < 1e-12, f"chunk {chunk}: carry mismatch"


def pin_step_matches_scan(orc, seed=8):
    """L chained one-token steps equal one scan over L, and a scan split at any token
    boundary (h_L1 fed back as h0) equals the whole scan. [SSM blog (shakilmahmud.com),
    section 3: recurrence at inference with constant memory]."""
    rng = _rng(seed)
    Bsz, L, Dm, N = 2, 11, 3, 4
    x = rng.standard_normal((Bsz, L, Dm)).astype(np.float32)
    dt = (0.5 * rng.standard_normal((Bsz, L, Dm))).astype(np.float32)
    z = rng.standard_normal((Bsz, L, Dm)).astype(np.float32)
    Bm = rng.standard_normal((Bsz, L, N)).astype(np.float32)
    Cm = rng.standard_normal((Bsz, L, N)).astype(np.float32)
    A = (-rng.uniform(0.5, 4.0, (Dm, N))).astype(np.float32)
    Dskip = rng.standard_normal(Dm).astype(np.float32)
    bias = rng.uniform(-3, 0, Dm).astype(np.float32)
    h0 = rng.standard_normal((Bsz, Dm, N)).astype(np.float32)
    y, hL = orc.scan(x, dt, A, Bm, Cm, D=Dskip, z=z, dt_bias=bias, h0=h0)
    h = h0.astype(np.float64).copy()
    for t in range(L):
        yt = orc.step(x[:, t], dt[:, t], A, Bm[:, t], Cm[:, t], h, D=Dskip, z=z[:, t], dt_bias=bias)
        assert _rel(yt - y[:, t], y[:, t]) < 1e-14, f"step {t} differs from the scan"
    assert _rel(h - hL, hL) < 1e-14
    L1 = 5
    y1, h1 = orc.scan(x[:, :L1], dt[:, :L1], A, Bm[:, :L1], Cm[:, :L1], D=Dskip, z=z[:, :L1],
                      dt_bias=bias, h0=h0)
    # h1 is float64; the scan takes a float32 initial state, so the split agrees to fp32 rounding.
    y2, h2 = orc.scan(x[:, L1:], dt[:, L1:], A, Bm[:, L1:], Cm[:, L1:], D=Dskip, z=z[:, L1:],
                      dt_bias=bias, h0=h1.astype(np.float32))
    assert _rel(np.concatenate([y1, y2], 1) - y, y) < 1e-6
    assert _rel(h2 - hL, hL) < 1e-6


def pin_no_input_dependence_on_future(orc, seed=9):
    """Causality: changing tokens at t >= T leaves y_t for t < T unchanged (bit for bit)."""
    rng = _rng(seed)
    Bsz, L, Dm, N = 1, 20, 3, 4
    args = [rng.standard_normal((Bsz, L, Dm)).astype(np.float32) for _ in range(3)]
    Bm = rng.standard_normal((Bsz, L, N)).astype(np.float32)
    Cm = rng.standard_normal((Bsz, L, N)).astype(np.float32)
    A = -np.tile(np.arange(1, N + 1, dtype=np.float32), (Dm, 1))
    y, _ = orc.scan(args[0], args[1], A, Bm, Cm, z=args[2])
    args2 = [a.copy() for a in args]
    for a in args2:
        a[:, 12:] = rng.standard_normal(a[:, 12:].shape)
    B2, C2 = Bm.copy(), Cm.copy()
    B2[:, 12:] += 1.0
    C2[:, 12:] -= 1.0
    y2, _ = orc.scan(args2[0], args2[1], A, B2, C2, z=args2[2])
    assert np.array_equal(y[:, :12], y2[:, :12]), "outputs before t must not depend on later tokens"
    assert not np.array_equal(y[:, 12:], y2[:, 12:])


ALL_PINS = [pin_lti_convolution, pin_theorem1_closed_form, pin_theorem1_gated_rnn,
            pin_small_delta_keeps_state, pin_large_delta_resets_state, pin_bruteforce,
            pin_associative_chunks, pin_step_matches_scan, pin_no_input_dependence_on_future]


def pin_lti_convolution_bf16(orc):
    pin_lti_convolution(orc, dtype="bf16", seed=11)


ALL_PINS.append(pin_lti_convolution_bf16)


def pin_conv_front_end(orc, dtype=DT_F32, seed=12, with_bias=True):
    """The block's short convolution in front of the SSM equals the SSM run on its output.

    [Mamba summary (azimuth.plus), block-architecture paragraph: main branch = projection,
    1-D convolution (kernel size 4), SiLU, selective SSM]. Expected input of the SSM:
    u = silu(v), v_t = conv_b + sum_k conv_w[k] x_{t-3+k}, computed per channel by numpy's
    cross-correlation over the sequence prefixed with conv_x0 (or three zeros); the oracle
    without the convolution is then run on u (stored as float32) with every other input
    unchanged, so the comparison carries only u's float32 rounding (~1e-7 relative).
    Checks: the taps' order and causality, the bias, the SiLU, the three tokens before
    t = 0 in both storage types, and that u feeds both Bbar x and D x.
    """
    rng = _rng(seed)
    Bsz, L, Dm, N = 2, 29, 5, 3
    xf = rng.standard_normal((Bsz, L, Dm)).astype(np.float32)
    x0f = rng.standard_normal((Bsz, 3, Dm)).astype(np.float32)
    toks = [rng.standard_normal((Bsz, L, Dm)).astype(np.float32) for _ in range(2)]  # dt, z
    BC = [rng.standard_normal((Bsz, L, N)).astype(np.float32) for _ in range(2)]
    A = (-0.2 - rng.random((Dm, N)) * 2.0).astype(np.float32)
    D = rng.standard_normal(Dm).astype(np.float32)
    bias = rng.standard_normal(Dm).astype(np.float32) * 0.5
    w = (rng.standard_normal((Dm, 4)) * 0.7).astype(np.float32)
    cb = (rng.standard_normal(Dm) * 0.3).astype(np.float32) if with_bias else None
    if dtype == "bf16":
        st = _bf16_bits
        val = _bf16_value
    else:
        st = lambda a: a
        val = lambda a: a.astype(np.float64)
    x, x0, dt, z, Bm, Cm = (st(a) for a in (xf, x0f, toks[0], toks[1], BC[0], BC[1]))
    for prefix in (x0, None):
        pre = val(prefix) if prefix is not None else np.zeros((Bsz, 3, Dm))
        seq = np.concatenate([pre, val(x)], axis=1)  # [Bsz, 3 + L, Dm]
        v = np.empty((Bsz, L, Dm))
        for b in range(Bsz):
            for d in range(Dm):
                v[b, :, d] = np.correlate(seq[b, :, d], w[d].astype(np.float64), mode="valid")
        if cb is not None:
            v += cb.astype(np.float64)
        u = (v * _sigma(v)).astype(np.float32)
        f32 = lambda a: val(a).astype(np.float32)  # exact: every stored value is a float32
        y_ref, h_ref = orc.scan(u, f32(dt), A, f32(Bm), f32(Cm), D=D, z=f32(z), dt_bias=bias, dtype=DT_F32)
        y, h = orc.scan(x, dt, A, Bm, Cm, D=D, z=z, dt_bias=bias, dtype=dtype, conv_w=w, conv_b=cb,
                        conv_x0=prefix)
        assert _rel(y - y_ref, y_ref) < 1e-5, "convolution front end: y"
        assert _rel(h - h_ref, h_ref) < 1e-5, "convolution front end: final state"


def pin_conv_front_end_bf16(orc):
    pin_conv_front_end(orc, dtype="bf16", seed=13, with_bias=False)


def pin_conv_step_matches_conv_scan(orc, seed=14):
    """Decode behind the short convolution: L chained steps, each reading the three previous
    tokens from a rolling window that starts as the scan's prefix, equal one scan with the
    convolution (itself pinned to numpy's cross-correlation above); the window ends as the
    last three tokens. [SSM blog (shakilmahmud.com), section 3: recurrence at inference;
    Mamba summary, block-architecture paragraph]."""
    rng = _rng(seed)
    Bsz, L, Dm, N = 2, 9, 3, 4
    x = rng.standard_normal((Bsz, L, Dm)).astype(np.float32)
    dt = (0.5 * rng.standard_normal((Bsz, L, Dm))).astype(np.float32)
    z = rng.standard_normal((Bsz, L, Dm)).astype(np.float32)
    Bm = rng.standard_normal((Bsz, L, N)).astype(np.float32)
    Cm = rng.standard_normal((Bsz, L, N)).astype(np.float32)
    A = (-rng.uniform(0.5, 4.0, (Dm, N))).astype(np.float32)
    Dskip = rng.standard_normal(Dm).astype(np.float32)
    bias = rng.uniform(-3, 0, Dm).astype(np.float32)
    w = (rng.standard_normal((Dm, 4)) * 0.7).astype(np.float32)
    cb = (rng.standard_normal(Dm) * 0.3).astype(np.float32)
    x0 = rng.standard_normal((Bsz, 3, Dm)).astype(np.float32)
    y, hL = orc.scan(x, dt, A, Bm, Cm, D=Dskip, z=z, dt_bias=bias, conv_w=w, conv_b=cb, conv_x0=x0)
    h = np.zeros((Bsz, Dm, N))
    window = x0.copy()
    for t in range(L):
        yt = orc.step(x[:, t], dt[:, t], A, Bm[:, t], Cm[:, t], h, D=Dskip, z=z[:, t], dt_bias=bias,
                      conv_w=w, conv_b=cb, conv_state=window)
        assert _rel(yt - y[:, t], y[:, t]) < 1e-14, f"convolution step {t} differs from the scan"
    assert _rel(h - hL, hL) < 1e-14
    assert np.array_equal(window, x[:, L - 3:]), "the window must end as the last three tokens"


ALL_PINS += [pin_conv_front_end, pin_conv_front_end_bf16, pin_conv_step_matches_conv_scan]


def _bwd_case(rng, Bsz, L, Dm, N, gate=True):
    f = lambda *shape: rng.standard_normal(shape).astype(np.float32)
    return dict(x=f(Bsz, L, Dm), dt=(0.7 * f(Bsz, L, Dm)).astype(np.float32), z=f(Bsz, L, Dm) if gate else None,
                B=f(Bsz, L, N), C=f(Bsz, L, N), A=(-0.2 - rng.random((Dm, N)) * 2.0).astype(np.float32),
                D=f(Dm), dt_bias=(0.5 * f(Dm)).astype(np.float32), h0=f(Bsz, Dm, N))


def pin_bwd_finite_differences(orc, seed=15, softplus=True, gate=True, exact_zoh=False, conv=False):
    """Every gradient of the backward equals the central difference of the forward.

    The loss is L = sum(dy * y) + sum(dh_last * h_L) with random dy, dh_last, so dL/dp is
    what the backward returns for dy, dh_last. Each input element p (float32) is moved by
    +-2^-12, exactly representable, and (L(p+) - L(p-)) / (p+ - p-) is compared with the
    gradient (truncation ~1e-7 relative at this step). A plain derivative check, by a
    route independent of the reverse sweep. exact_zoh and conv (the short convolution,
    with bias and the three tokens before the sequence) select those forward variants; the
    convolution's taps, bias and prefix tokens are then differentiated too."""
    rng = _rng(seed)
    Bsz, L, Dm, N = 2, 6, 3, 3
    inp = _bwd_case(rng, Bsz, L, Dm, N, gate)
    if exact_zoh:
        # A spanning the exact hold's regimes: tiny |Delta A| (the series branch of dw/dA),
        # exactly zero (w = Delta), and ordinary values
        inp["A"][0, 0], inp["A"][1, 1], inp["A"][2, 2] = np.float32(-1e-3), np.float32(0.0), np.float32(3e-4)
    cv = {}
    if conv:
        cv = dict(conv_w=(rng.random((Dm, 4)) - 0.5).astype(np.float32),
                  conv_b=(rng.random(Dm) - 0.5).astype(np.float32),
                  conv_x0=rng.standard_normal((Bsz, 3, Dm)).astype(np.float32))
        inp.update(cv)
    dy = rng.standard_normal((Bsz, L, Dm)).astype(np.float32)
    dh_last = rng.standard_normal((Bsz, Dm, N))

    def loss(v):
        kw = {k: v[k] for k in cv}
        y, h = orc.scan(v["x"], v["dt"], v["A"], v["B"], v["C"], D=v["D"], z=v["z"], dt_bias=v["dt_bias"],
                        h0=v["h0"], delta_softplus=softplus, exact_zoh=exact_zoh, **kw)
        return float(np.sum(dy * y) + np.sum(dh_last * h))

    g = orc.scan_bwd(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], dy, D=inp["D"], z=inp["z"],
                     dt_bias=inp["dt_bias"], h0=inp["h0"], dh_last=dh_last, delta_softplus=softplus,
                     exact_zoh=exact_zoh, **cv)
    names = {"x": "dx", "dt": "ddt", "z": "dz", "B": "dB", "C": "dC", "A": "dA", "D": "dD",
             "dt_bias": "ddt_bias", "h0": "dh0"}
    if conv:
        names.update(conv_w="dconv_w", conv_b="dconv_b", conv_x0="dconv_x0")
    step = np.float32(2.0 ** -12)
    for key, gname in names.items():
        if inp[key] is None:
            assert g[gname] is None
            continue
        fd = np.empty(inp[key].shape)
        for idx in np.ndindex(inp[key].shape):
            p0 = inp[key][idx]
            hi, lo = np.float32(p0 + step), np.float32(p0 - step)
            inp[key][idx] = hi
            up = loss(inp)
            inp[key][idx] = lo
            down = loss(inp)
            inp[key][idx] = p0
            fd[idx] = (up - down) / (float(hi) - float(lo))
        assert _rel(g[gname] - fd, fd) < 2e-5, f"backward {gname} differs from the central difference"


def pin_bwd_finite_differences_plain(orc):
    """The same without softplus and without the gate."""
    pin_bwd_finite_differences(orc, seed=16, softplus=False, gate=False)


def pin_bwd_bf16_storage(orc, seed=17):
    """bfloat16 storage is read as its exact float32 values, dy included."""
    rng = _rng(seed)
    inp = _bwd_case(rng, 2, 9, 4, 3)
    dy = rng.standard_normal((2, 9, 4)).astype(np.float32)
    toks = ("x", "dt", "z", "B", "C")
    bits = {k: _bf16_bits(inp[k]) for k in toks}
    vals = {k: _bf16_value(bits[k]).astype(np.float32) for k in toks}
    dyb = _bf16_bits(dy)
    g16 = orc.scan_bwd(bits["x"], bits["dt"], inp["A"], bits["B"], bits["C"], dyb, D=inp["D"], z=bits["z"],
                       dt_bias=inp["dt_bias"], h0=inp["h0"], dtype="bf16")
    g32 = orc.scan_bwd(vals["x"], vals["dt"], inp["A"], vals["B"], vals["C"],
                       _bf16_value(dyb).astype(np.float32), D=inp["D"], z=vals["z"], dt_bias=inp["dt_bias"],
                       h0=inp["h0"])
    for k in g32:
        assert np.array_equal(g16[k], g32[k]), f"bf16 backward {k} differs"


def pin_bwd_finite_differences_zoh(orc):
    """The backward of the exact zero-order hold, against the central difference."""
    pin_bwd_finite_differences(orc, seed=20, exact_zoh=True)


def pin_bwd_finite_differences_conv(orc):
    """The backward through the short convolution (taps, bias, prefix tokens and the raw
    tokens), against the central difference."""
    pin_bwd_finite_differences(orc, seed=21, conv=True)


def pin_bwd_finite_differences_zoh_conv(orc):
    """Both variants at once, without softplus."""
    pin_bwd_finite_differences(orc, seed=22, softplus=False, exact_zoh=True, conv=True)


def pin_zoh_weight_series_matches_closed_form(orc, seed=23):
    """dL/dA of the exact hold on both sides of |Delta A| = 0.25, where the oracle switches
    between the closed form of dw/dA and its series: for A in {-0.05, -0.2, -0.3, -1.5}
    (with Delta about 0.3 to 1.5) it equals the central difference of the loss in A, with
    a step of 2^-14 and a tolerance of 1e-6."""
    rng = _rng(seed)
    Bsz, L, Dm, N = 1, 5, 1, 2
    inp = _bwd_case(rng, Bsz, L, Dm, N, gate=False)
    dy = rng.standard_normal((Bsz, L, Dm)).astype(np.float32)
    for a in (-0.05, -0.2, -0.3, -1.5):  # Delta ~ 0.5..1.5 puts Delta A on both sides of 0.25
        inp["A"][0, :] = np.float32(a)
        g = orc.scan_bwd(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], dy, D=inp["D"],
                         dt_bias=inp["dt_bias"], h0=inp["h0"], exact_zoh=True)["dA"]

        def loss(A):
            y, _ = orc.scan(inp["x"], inp["dt"], A, inp["B"], inp["C"], D=inp["D"], dt_bias=inp["dt_bias"],
                            h0=inp["h0"], exact_zoh=True)
            return float(np.sum(dy * y))
        for n in range(N):
            A1, A2 = inp["A"].copy(), inp["A"].copy()
            st = np.float32(2.0 ** -14)
            A1[0, n] += st
            A2[0, n] -= st
            fd = (loss(A1) - loss(A2)) / (float(A1[0, n]) - float(A2[0, n]))
            assert abs(g[0, n] - fd) <= 1e-6 * max(1.0, abs(fd)), f"dA at A = {a} differs from the central difference"


ALL_PINS += [pin_bwd_finite_differences, pin_bwd_finite_differences_plain, pin_bwd_bf16_storage,
             pin_bwd_finite_differences_zoh, pin_bwd_finite_differences_conv, pin_bwd_finite_differences_zoh_conv,
             pin_zoh_weight_series_matches_closed_form]


def pin_ssd_semiseparable_form(orc, seed=18):
    """With one scalar A per channel (A[d, n] = a_d for every n, the Mamba-2 restriction), the
    scan equals multiplication by a lower-triangular semiseparable matrix:
    y_t = sum_{s<=t} (C_t . B_s) exp(a_d (S_t - S_s)) Delta_s x_s + exp(a_d S_t) C_t . h0,
    S_t = Delta_1 + ... + Delta_t (the structured state space duality of the Mamba-2 article,
    mugbit.ir, "Mamba-2 and SSD" section: the recurrence as a structured matrix product).
    The matrix is formed with numpy and applied as one product, independently of the
    oracle's loop."""
    rng = _rng(seed)
    Bsz, L, Dm, N = 2, 23, 3, 4
    x = rng.standard_normal((Bsz, L, Dm)).astype(np.float32)
    dt = (0.5 * rng.standard_normal((Bsz, L, Dm))).astype(np.float32)
    Bm = rng.standard_normal((Bsz, L, N)).astype(np.float32)
    Cm = rng.standard_normal((Bsz, L, N)).astype(np.float32)
    a = (-0.3 - rng.random(Dm) * 2.0).astype(np.float32)
    A = np.repeat(a[:, None], N, axis=1)
    bias = (0.3 * rng.standard_normal(Dm)).astype(np.float32)
    h0 = rng.standard_normal((Bsz, Dm, N)).astype(np.float32)
    y, _ = orc.scan(x, dt, A, Bm, Cm, dt_bias=bias, h0=h0)
    delta = _softplus(dt.astype(np.float64) + bias.astype(np.float64))       # [Bsz, L, Dm]
    S = np.cumsum(delta, axis=1)
    ref = np.empty((Bsz, L, Dm))
    tri = np.tril(np.ones((L, L), dtype=bool))
    for b in range(Bsz):
        CB = Cm[b].astype(np.float64) @ Bm[b].astype(np.float64).T            # [L, L]: C_t . B_s
        for d in range(Dm):
            decay = np.where(tri, np.exp(a[d] * (S[b, :, d][:, None] - S[b, :, d][None, :])), 0.0)
            M = CB * decay                                                     # the semiseparable matrix
            u = delta[b, :, d] * x[b, :, d]
            ref[b, :, d] = M @ u + np.exp(a[d] * S[b, :, d]) * (Cm[b].astype(np.float64) @ h0[b, d].astype(np.float64))
    assert _rel(y - ref, ref) < 1e-11, "scalar-A scan differs from its semiseparable matrix form"


ALL_PINS.append(pin_ssd_semiseparable_form)


def pin_segment_affine_maps(orc, seed=19):
    """Across a segment of the sequence both recurrences are affine with the same slope
    P = exp(A sum_t Delta_t): the end state is P h_start + (the end state from a zero
    start), and the adjoint passed out of the segment's start is P g_end + (the one from a
    zero g_end). This is what lets a segment's work start before its neighbours' is done
    (Mamba summary, hardware-aware algorithm paragraph: the parallel scan). Checked on the
    oracle's forward (h_L against h0) and backward (dh0 against dh_last) by superposition."""
    rng = _rng(seed)
    inp = _bwd_case(rng, 2, 17, 3, 4)
    dy = rng.standard_normal((2, 17, 3)).astype(np.float32)
    g_end = rng.standard_normal((2, 3, 4))
    P = np.exp(inp["A"].astype(np.float64)[None] *
               _softplus(inp["dt"].astype(np.float64) + inp["dt_bias"].astype(np.float64)).sum(axis=1)[:, :, None])
    args = (inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"])
    kw = dict(D=inp["D"], z=inp["z"], dt_bias=inp["dt_bias"])
    _, h_full = orc.scan(*args, h0=inp["h0"], **kw)
    _, h_zero = orc.scan(*args, **kw)
    assert _rel(h_full - (P * inp["h0"] + h_zero), h_full) < 1e-12, "forward: end state not affine in h0"
    g_full = orc.scan_bwd(*args, dy, dh_last=g_end, h0=inp["h0"], **kw)["dh0"]
    g_zero = orc.scan_bwd(*args, dy, h0=inp["h0"], **kw)["dh0"]
    assert _rel(g_full - (P * g_end + g_zero), g_full) < 1e-12, "backward: start adjoint not affine in dh_last"


ALL_PINS.append(pin_segment_affine_maps)
