"""Pins of the oracle's shard step against closed forms, fp64 textbook values
and special cases.  The pages name Adam and its 12 bytes of fp32 state
("ZeRO memory optimization: training large models", trishampatil.com, "The
Real Problem") but print no update equations; the reading pinned here is
Kingma & Ba (2015), Algorithm 1, with decoupled weight decay (Loshchilov &
Hutter 2019)."""
import math

import numpy as np
import pytest

import oracle
from zero_dp_partitioned_shard_b200 import synth

F32 = np.float32


def _const_grads(g_target, nd, S):
    """fp16 contributions [nd, n] whose rank sum / S is exactly g_target."""
    g_target = np.asarray(g_target, dtype=np.float64)
    share = g_target * S / nd
    c = share.astype(np.float16)
    G = np.repeat(c[None, :], nd, axis=0)
    g = G.astype(np.float64).sum(axis=0) / S
    assert np.array_equal(g.astype(np.float32).astype(np.float64), g), "setup must be exact"
    return G.view(np.uint16), g


def _run(G, p0, hp, steps, m0=None, v0=None):
    n = G.shape[1]
    master = p0.astype(np.float32).copy()
    m = np.zeros(n, F32) if m0 is None else m0.copy()
    v = np.zeros(n, F32) if v0 is None else v0.copy()
    P = np.zeros(n, np.uint16)
    opt = oracle.Opt()
    infos = []
    for _ in range(steps):
        infos.append(oracle.step(G, master, m, v, P, hp, opt))
    return master, m, v, P, opt, infos


@pytest.mark.parametrize("wd", [0.0, 0.01])
def test_constant_gradient_closed_form(wd):
    # |g| spans 1e-6 (where eps = 1e-8 is a 1 % effect) to 4
    rs = np.random.default_rng(11)
    mags = np.array([2.0 ** k for k in range(-20, 3)])
    g_t = np.concatenate([mags, -mags, mags * 1.5])
    nd, S, T = 4, 1024.0, 5
    G, g = _const_grads(g_t, nd, S)
    p0 = synth.normal_f32(g.size, seed=3, std=0.02).astype(np.float64)
    hp = oracle.HP(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=wd, loss_scale=S)
    master, m, v, P, opt, infos = _run(G, p0, hp, T)
    b1, b2 = float(F32(0.9)), float(F32(0.999))
    # m_t = (1 - b1^t) g and v_t = (1 - b2^t) g^2 exactly in real arithmetic
    m_exact = (1 - b1 ** T) * g
    v_exact = (1 - b2 ** T) * g * g
    assert np.all(np.abs(m - m_exact) <= 8 * T * np.spacing(np.abs(m_exact).astype(F32)))
    assert np.all(np.abs(v - v_exact) <= 8 * T * np.spacing(np.abs(v_exact).astype(F32)))
    # bias-corrected moments are g and g^2, so each step moves p by lr*u
    lr = float(F32(1e-3))
    u = lr * g / (np.abs(g) + float(F32(1e-8)))
    if wd == 0.0:
        p_exact = p0 - T * u
    else:
        a = 1.0 - float(F32(lr * float(F32(wd))))
        p_exact = a ** T * p0 - u * (1 - a ** T) / (1 - a)
    tol = T * (2 * np.spacing(np.abs(p_exact).astype(F32)).astype(np.float64) + 4e-7 * np.abs(u))
    assert np.all(np.abs(master - p_exact) <= tol), np.max(np.abs(master - p_exact) / tol)
    assert opt.t == T
    assert np.array_equal(P, master.astype(np.float16).view(np.uint16))


def test_zero_gradient_leaves_parameters():
    nd, n = 3, 100
    G = np.zeros((nd, n), np.uint16)
    p0 = synth.normal_f32(n, seed=1, std=0.02)
    hp = oracle.HP(loss_scale=1.0)
    master, m, v, P, opt, infos = _run(G, p0, hp, 3)
    assert np.array_equal(master, p0) and (m == 0).all() and (v == 0).all()
    assert infos[-1]["grad_norm"] == 0.0 and opt.t == 3


def _adam_fp64(gs, p0, lr, b1, b2, eps, wd):
    """Textbook Adam/AdamW in fp64 (Kingma & Ba 2015, Alg. 1)."""
    p, m, v = p0.copy(), np.zeros_like(p0), np.zeros_like(p0)
    for t, g in enumerate(gs, start=1):
        p_old = p.copy()
        m = b1 * m + (1 - b1) * g
        v = b2 * v + (1 - b2) * g * g
        mh = m / (1 - b1 ** t)
        vh = v / (1 - b2 ** t)
        p = p_old - lr * wd * p_old - lr * mh / (np.sqrt(vh) + eps)
    return p, m, v


def test_random_gradients_match_fp64_textbook_within_rounding():
    nd, n, S, T = 8, 4096, 65536.0, 6
    hp = oracle.HP(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01, loss_scale=S)
    p0 = synth.normal_f32(n, seed=2, std=0.02)
    master, m, v = p0.copy(), np.zeros(n, F32), np.zeros(n, F32)
    P = np.zeros(n, np.uint16)
    opt = oracle.Opt()
    gs = []
    for t in range(T):
        G = synth.grads_f16(nd, n, seed=100 + t, std=1e-3, scale=S)
        gs.append(G.view(np.float16).astype(np.float64).sum(axis=0) / S)
        oracle.step(G, master, m, v, P, hp, opt)
    c = lambda x: float(F32(x))
    p64, m64, v64 = _adam_fp64(gs, p0.astype(np.float64), c(1e-3), c(0.9), c(0.999), c(1e-8),
                               c(0.01))
    # m can cancel to near zero: bound its error by the same recurrence on |g|
    _, m_abs, _ = _adam_fp64([np.abs(g) for g in gs], p0.astype(np.float64), c(1e-3), c(0.9),
                             c(0.999), c(1e-8), c(0.01))
    assert np.max(np.abs(m - m64) / m_abs) < 1e-6
    assert np.max(np.abs(v - v64) / np.abs(v64)) < 1e-6
    assert np.max(np.abs(master - p64)) < 5e-8


def test_clip_coefficient_and_norm_exact_case():
    # Psi = 1024 elements all equal to g = 2^-10 after the reduction:
    # ||g|| = 32 * 2^-10 = 2^-5 exactly; clipping at 2^-6 halves every element
    nd, n, S = 4, 1024, 1024.0
    G, g = _const_grads(np.full(n, 2.0 ** -10), nd, S)
    p0 = synth.normal_f32(n, seed=4, std=0.02)
    hp = oracle.HP(loss_scale=S, max_grad_norm=2.0 ** -6)
    master, m, v, P, opt, infos = _run(G, p0, hp, 1)
    assert infos[0]["grad_norm"] == 2.0 ** -5 and infos[0]["sumsq"] == 2.0 ** -10
    assert infos[0]["clip_coef"] == 0.5
    assert (m == F32(1.0 - F32(0.9)) * F32(2.0 ** -11)).all()
    assert (v == F32(1.0 - F32(0.999)) * F32(2.0 ** -22)).all()
    # below the threshold nothing is scaled
    hp2 = oracle.HP(loss_scale=S, max_grad_norm=1.0)
    _, m2, _, _, _, infos2 = _run(G, p0, hp2, 1)
    assert infos2[0]["clip_coef"] == 1.0
    assert (m2 == F32(1.0 - F32(0.9)) * F32(2.0 ** -10)).all()


@pytest.mark.parametrize("nd,psi,S,c", [(4, 1_000, 1024.0, 0.5), (16, 4_096, 65536.0, 3.0),
                                        (1, 7, 1.0, -2.0)])
def test_norm_of_constant_contributions(nd, psi, S, c):
    G = np.full((nd, psi), np.float16(c)).view(np.uint16)
    hp = oracle.HP(loss_scale=S)
    _, _, _, _, _, infos = _run(G, np.zeros(psi, F32), hp, 1)
    want = nd * abs(c) * math.sqrt(psi) / S
    assert abs(infos[0]["grad_norm"] - want) <= 2 * math.ulp(want)
    s, bad = oracle.grad_sumsq(G, hp)
    assert s == infos[0]["sumsq"] and not bad


def test_norm_is_the_exact_sum_of_squares():
    """The oracle's sum of squares equals the exactly rounded sum (math.fsum)
    of the exact fp64 squares of the fp32 reduced gradient, to 2 ulp, even
    over many terms of mixed magnitude, where a left-to-right fp64 sum drifts."""
    nd, n, S = 4, 1 << 20, 1024.0
    G = synth.grads_f16(nd, n, seed=31, std=1e-3, scale=S)
    G[:, ::977] = np.float16(1000.0).view(np.uint16)   # a few large terms
    g = oracle.all_reduce(G, n) * np.float32(1.0 / S)    # fp32, as the step unscales
    exact = math.fsum((g.astype(np.float64) ** 2).tolist())
    hp = oracle.HP(loss_scale=S)
    s, bad = oracle.grad_sumsq(G, hp)
    assert not bad and abs(s - exact) <= 2 * math.ulp(exact)
    _, _, _, _, _, infos = _run(G, np.zeros(n, F32), hp, 1)
    assert abs(infos[0]["sumsq"] - exact) <= 2 * math.ulp(exact)
    assert infos[0]["grad_norm"] == math.sqrt(infos[0]["sumsq"])


def test_streamed_sum_of_squares_carries_its_compensation():
    """Pieces streamed with one carried accumulator give the single-pass sum
    bit for bit; pieces with their own accumulators, added exactly
    (math.fsum of every sum and compensation term), stay within 2 ulp of the
    exactly rounded sum of the exact squares."""
    nd, n, S = 3, 300_007, 64.0
    G = synth.grads_f16(nd, n, seed=33, std=1e-2, scale=S)
    G[:, ::613] = np.float16(3000.0).view(np.uint16)
    hp = oracle.HP(loss_scale=S)
    whole, _ = oracle.grad_sumsq(G, hp)
    cuts = [0, 1, 4097, 100_000, 100_001, 250_000, n]
    carried = np.zeros(2, np.float64)
    separate = []
    for a, b in zip(cuts[:-1], cuts[1:]):
        oracle.grad_sumsq(np.ascontiguousarray(G[:, a:b]), hp, carried)
        own = np.zeros(2, np.float64)
        oracle.grad_sumsq(np.ascontiguousarray(G[:, a:b]), hp, own)
        separate += own.tolist()
    assert carried.sum() == whole and carried[0] + carried[1] == whole
    g = oracle.all_reduce(G, n) * np.float32(1.0 / S)
    exact = math.fsum((g.astype(np.float64) ** 2).tolist())
    assert abs(math.fsum(separate) - exact) <= 2 * math.ulp(exact)


def test_average_over_nd_divides_by_nd():
    nd, n, S = 8, 64, 1024.0
    G, g = _const_grads(np.full(n, 2.0 ** -8), nd, S)
    hp = oracle.HP(loss_scale=S, average_over_nd=True)
    _, m, _, _, _, infos = _run(G, np.zeros(n, F32), hp, 1)
    assert infos[0]["grad_norm"] == pytest.approx(math.sqrt(n) * 2.0 ** -11, rel=1e-15)
    assert (m == F32(1.0 - F32(0.9)) * F32(2.0 ** -11)).all()


def _snapshot(*arrs):
    return [a.copy() for a in arrs]


@pytest.mark.parametrize("case", ["inf_one_rank", "pos_neg_inf_nan", "nan", "sum_overflow"])
def test_overflow_skips_everything(case):
    nd, n, S = 4, 1000, 1024.0
    G = synth.grads_f16(nd, n, seed=9, std=1e-3, scale=S).copy()
    if case == "inf_one_rank":
        G[2, 517] = 0x7C00
    elif case == "pos_neg_inf_nan":
        G[0, 3] = 0x7C00
        G[3, 3] = 0xFC00
    elif case == "nan":
        G[1, 999] = 0x7E00
    else:
        # a loss scale below 1 makes the unscaled value leave fp32's range
        G[:, 10] = np.float16(65504.0).view(np.uint16)
    if case == "sum_overflow":
        S = 2.0 ** -120
    hp = oracle.HP(loss_scale=S, max_grad_norm=1.0)
    master = synth.normal_f32(n, seed=1, std=0.02)
    m = synth.normal_f32(n, seed=2, std=1e-4)
    v = np.abs(synth.normal_f32(n, seed=3, std=1e-6))
    P = master.astype(np.float16).view(np.uint16).copy()
    opt = oracle.Opt(t=5, beta1_pow=0.9 ** 5, beta2_pow=0.999 ** 5)
    before = _snapshot(master, m, v, P)
    info = oracle.step(G, master, m, v, P, hp, opt)
    assert info["overflow"] == 1
    for a, b in zip(before, (master, m, v, P)):
        assert np.array_equal(a.view(np.uint8), b.view(np.uint8))
    assert (opt.t, opt.beta1_pow, opt.beta2_pow) == (5, 0.9 ** 5, 0.999 ** 5)


def test_non_finite_pad_is_ignored():
    nd, psi, S = 4, 1001, 1024.0
    p = oracle.plan(psi, nd, 256)
    G = synth.grads_f16(nd, psi, seed=8, std=1e-3, scale=S, stride=p.psi_pad, pad_fill=np.inf)
    hp = oracle.HP(loss_scale=S)
    master = synth.normal_f32(psi, seed=1, std=0.02)
    info = oracle.step(G, master, np.zeros(psi, F32), np.zeros(psi, F32),
                       np.zeros(psi, np.uint16), hp, oracle.Opt())
    assert info["overflow"] == 0 and math.isfinite(info["grad_norm"])


def test_bias_corrections_running_products():
    hp = oracle.HP(beta1=0.9, beta2=0.999)
    opt = oracle.Opt()
    b1, b2 = float(F32(0.9)), float(F32(0.999))
    for t in range(1, 2001):
        p1, p2, c1, c2 = oracle.bias_corrections(hp, opt)
        assert p1 == pytest.approx(b1 ** t, rel=4e-16 * t)
        assert p2 == pytest.approx(b2 ** t, rel=4e-16 * t)
        assert c1 == F32(1.0 - p1) and c2 == F32(1.0 - p2)
        opt = oracle.Opt(t, p1, p2)


def test_owner_by_owner_update_equals_flat_step():
    """Each owner updating only its slice, with the global clip coefficient and
    bias corrections, reproduces the flat step bit for bit."""
    nd, psi, S = 5, 3001, 1024.0
    p = oracle.plan(psi, nd, 8)
    G = synth.grads_f16(nd, psi, seed=21, std=1e-3, scale=S, stride=p.psi_pad)
    hp = oracle.HP(loss_scale=S, max_grad_norm=1e-3, weight_decay=0.01)
    master = synth.normal_f32(psi, seed=1, std=0.02)
    m = synth.normal_f32(psi, seed=2, std=1e-5)
    v = np.abs(synth.normal_f32(psi, seed=3, std=1e-8))
    opt = oracle.Opt(t=2, beta1_pow=float(F32(0.9)) ** 2, beta2_pow=float(F32(0.999)) ** 2)
    flat = _snapshot(master, m, v) + [np.zeros(psi, np.uint16)]
    _, _, c1, c2 = oracle.bias_corrections(hp, opt)
    info = oracle.step(G, *flat, hp, oracle.Opt(opt.t, opt.beta1_pow, opt.beta2_pow))
    assert info["clip_coef"] < 1.0
    P = np.zeros(psi, np.uint16)
    for r in range(nd):
        s, n = p.shard(r)
        if n == 0:
            continue
        sl = slice(s, s + n)
        mm, mo, vo, po = master[sl].copy(), m[sl].copy(), v[sl].copy(), P[sl].copy()
        oracle.update_elements(G[:, sl], mm, mo, vo, po, hp, info["clip_coef"], c1, c2)
        master[sl], m[sl], v[sl], P[sl] = mm, mo, vo, po
    for a, b in zip((master, m, v, P), flat):
        assert np.array_equal(a.view(np.uint8), b.view(np.uint8))


def test_threads_do_not_change_results():
    nd, psi, S = 8, 20_000, 65536.0
    G = synth.grads_f16(nd, psi, seed=5, std=1e-3, scale=S)
    hp = oracle.HP(loss_scale=S, weight_decay=0.01, max_grad_norm=1e-3)
    outs = []
    for th in (1, 4):
        master = synth.normal_f32(psi, seed=1, std=0.02)
        m, v, P = np.zeros(psi, F32), np.zeros(psi, F32), np.zeros(psi, np.uint16)
        oracle.step(G, master, m, v, P, hp, oracle.Opt(), threads=th)
        outs.append((master, m, v, P))
    for a, b in zip(*outs):
        assert np.array_equal(a.view(np.uint8), b.view(np.uint8))


def test_dynamic_loss_scale_state_machine():
    """Dynamic loss scaling (Micikevicius et al. 2018, sec. 3.2; the pages
    cite the paper as background only): halve on a skipped step, double after
    growth_interval consecutive applied steps, counting restarts on change."""
    nd, n, S0 = 2, 256, 2.0 ** 16
    G_ok = synth.grads_f16(nd, n, seed=71, std=1e-3, scale=S0)
    G_bad = G_ok.copy()
    G_bad[1, 7] = 0x7C00
    hp = oracle.HP(loss_scale=1.0)   # ignored while the dynamic scale is in use
    opt = oracle.Opt(loss_scale=S0, growth_interval=3, growth_factor=2.0, backoff_factor=0.5)
    master = synth.normal_f32(n, seed=72, std=0.02)
    m, v, P = np.zeros(n, F32), np.zeros(n, F32), np.zeros(n, np.uint16)
    plan = ["ok", "ok", "ok", "ok", "ok", "bad", "ok", "bad", "bad", "ok", "ok", "ok"]
    want = [(S0, 1), (S0, 2), (2 * S0, 0), (2 * S0, 1), (2 * S0, 2), (S0, 0), (S0, 1),
            (S0 / 2, 0), (S0 / 4, 0), (S0 / 4, 1), (S0 / 4, 2), (S0 / 2, 0)]
    for kind, (s_after, good_after) in zip(plan, want):
        info = oracle.step(G_bad if kind == "bad" else G_ok, master, m, v, P, hp, opt)
        assert info["overflow"] == (kind == "bad")
        assert (opt.loss_scale, opt.good_steps) == (s_after, good_after)
    assert opt.t == plan.count("ok")


def test_dynamic_scale_replaces_the_static_one():
    nd, n, S = 4, 1000, 2.0 ** 10
    G = synth.grads_f16(nd, n, seed=73, std=1e-3, scale=S)
    outs = []
    for opt, hp in ((oracle.Opt(loss_scale=S), oracle.HP(loss_scale=7.0)),
                    (oracle.Opt(), oracle.HP(loss_scale=S))):
        master = synth.normal_f32(n, seed=74, std=0.02)
        m, v, P = np.zeros(n, F32), np.zeros(n, F32), np.zeros(n, np.uint16)
        oracle.step(G, master, m, v, P, hp, opt)
        outs.append((master, m, v, P))
    for a, b in zip(*outs):
        assert np.array_equal(a.view(np.uint8), b.view(np.uint8))


def test_static_scale_leaves_the_scale_state_alone():
    G = synth.grads_f16(2, 100, seed=75, std=1e-3, scale=8.0)
    opt = oracle.Opt()
    oracle.step(G, synth.normal_f32(100, seed=1, std=0.02), np.zeros(100, F32), np.zeros(100, F32),
                np.zeros(100, np.uint16), oracle.HP(loss_scale=8.0), opt)
    assert (opt.loss_scale, opt.good_steps, opt.t) == (0.0, 0, 1)


def test_bf16_storage_step_matches_its_definition():
    """With bf16 gradients and parameters the step is the same arithmetic with
    bf16 widening of the contributions and a bf16 cast of the master."""
    nd, n, S = 4, 2000, 1.0
    G32 = (synth.normal_f32(nd * n, seed=91, std=1e-3) * np.float32(S)).reshape(nd, n)
    G = oracle.float_to_bf16(G32)
    hp = oracle.HP(loss_scale=S, weight_decay=0.01, storage=1)
    master = synth.normal_f32(n, seed=92, std=0.02)
    m, v, P = np.zeros(n, F32), np.zeros(n, F32), np.zeros(n, np.uint16)
    m0 = master.copy()
    oracle.step(G, master, m, v, P, hp, oracle.Opt())
    # the reduced gradient is the rank-order fp32 sum of the widened bf16 values
    g = oracle.bf16_to_float(G[0])
    for r in range(1, nd):
        g = (g + oracle.bf16_to_float(G[r])).astype(F32)
    assert (m == (F32(1.0 - F32(0.9)) * g).astype(F32)).all()
    assert np.array_equal(P, oracle.float_to_bf16(master))
    assert not np.array_equal(master, m0)
