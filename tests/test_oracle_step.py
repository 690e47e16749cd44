"""Pins for the oracle's optimizer step (CPU only).

The abstract of "8-bit Optimizers via Block-wise Quantization" (reproduced on the blog.csdn.net
bitsandbytes guide, section 2) names the stateful optimizers -- SGD with momentum (smoothed
sum) and Adam (smoothed and squared sums) -- and presents the 8-bit versions as substitutes
that need no other change and behave as the 32-bit ones.  The page "bitsandbytes深度解析", section
"优化器模块深度分析", lists AdamW8bit, Adam8bit, SGD8bit and Lion8bit.  So with quantization
out of the way (32-bit state) the oracle's step must agree with torch.optim's AdamW, Adam and
SGD, which these tests run in float64 as an independent reference; Lion is pinned by its
closed-form special cases.  The 8-bit path is pinned as "dequantize -> the same update ->
nearest-code requantize" against torch and an exact brute-force nearest code.
"""

import numpy as np
import pytest
import torch
from hypothesis import given, settings, strategies as st

HP = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01)


def _f(x):
    """binary32 value of a hyper-parameter, as the oracle sees it."""
    return float(np.float32(x))


def _close(got, want, scale, rtol=2e-6, ulps=4):
    """|got - want| <= rtol*|want| + ulps * ulp32(scale): fp32 rounding against an fp64 reference,
    with an absolute floor set by the size of the operands (cancellation leaves small results)."""
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    tol = rtol * np.abs(want) + ulps * np.spacing(np.abs(np.asarray(scale, np.float32))).astype(np.float64)
    bad = np.abs(got - want) > tol
    assert not bad.any(), (np.nonzero(bad)[0][:5], got[bad][:5], want[bad][:5])


def _grads(n, steps, seed, tiny_fraction=0.05):
    rng = np.random.default_rng(seed)
    gs = []
    for _ in range(steps):
        g = (rng.standard_normal(n) * 1e-3).astype(np.float32)
        tiny = rng.random(n) < tiny_fraction  # gradients where eps matters
        g[tiny] *= 1e-5
        gs.append(g)
    return gs


def _torch_run(opt_cls, p0, grads, **kw):
    p = torch.nn.Parameter(torch.from_numpy(p0.astype(np.float64)))
    opt = opt_cls([p], **kw)
    for g in grads:
        p.grad = torch.from_numpy(g.astype(np.float64))
        opt.step()
    return p.detach().numpy(), opt.state[p]


@pytest.mark.parametrize("wd", [0.0, 0.01])
def test_adamw_32bit_matches_torch(oracle_mod, wd):
    n, steps = 5000, 10
    p0 = (np.random.default_rng(0).standard_normal(n) * 0.02).astype(np.float32)
    grads = _grads(n, steps, 1)
    p = p0.copy()
    m = np.zeros(n, np.float32)
    v = np.zeros(n, np.float32)
    hp = dict(HP, weight_decay=wd)
    for t, g in enumerate(grads, 1):
        oracle_mod.step_tensor("adamw", p, g, m, v, None, None, None, None, 2048, step=t, **hp)
    pt, st = _torch_run(torch.optim.AdamW, p0, grads, lr=_f(hp["lr"]), betas=(_f(0.9), _f(0.999)),
                        eps=_f(1e-8), weight_decay=_f(wd), foreach=False)
    _close(p, pt, np.abs(p0) + hp["lr"] * steps)  # operand scale: p0 and the summed updates
    _close(m, st["exp_avg"].numpy(), np.max(np.abs(m)), rtol=2e-5)
    _close(v, st["exp_avg_sq"].numpy(), np.max(v), rtol=2e-5)


def test_adamw_first_step_closed_form(oracle_mod):
    """P5: from zero state, step 1 moves p by lr * g / (|g| + eps) after the decoupled decay."""
    n = 4096
    rng = np.random.default_rng(5)
    p0 = (rng.standard_normal(n) * 0.02).astype(np.float32)
    g = (rng.standard_normal(n) * 1e-3).astype(np.float32)
    p = p0.copy()
    m = np.zeros(n, np.float32)
    v = np.zeros(n, np.float32)
    oracle_mod.step_tensor("adamw", p, g, m, v, None, None, None, None, 2048, step=1, **HP)
    lr, wd, eps = _f(HP["lr"]), _f(HP["weight_decay"]), _f(HP["eps"])
    g64 = g.astype(np.float64)
    want = p0 * (1 - lr * wd) - lr * g64 / (np.abs(g64) + eps)
    _close(p, want, np.abs(p0) + lr, rtol=0)


def test_adam_l2_matches_torch(oracle_mod):
    n, steps = 3000, 6
    p0 = (np.random.default_rng(2).standard_normal(n) * 0.02).astype(np.float32)
    grads = _grads(n, steps, 3)
    p = p0.copy()
    m = np.zeros(n, np.float32)
    v = np.zeros(n, np.float32)
    hp = dict(HP, weight_decay=0.1)
    for t, g in enumerate(grads, 1):
        oracle_mod.step_tensor("adam", p, g, m, v, None, None, None, None, 256, step=t, **hp)
    pt, _ = _torch_run(torch.optim.Adam, p0, grads, lr=_f(1e-3), betas=(_f(0.9), _f(0.999)), eps=_f(1e-8),
                       weight_decay=_f(0.1), foreach=False)
    _close(p, pt, np.abs(p0) + 1e-3 * steps)


@pytest.mark.parametrize("wd", [0.0, 1e-2])
def test_momentum_matches_torch_sgd(oracle_mod, wd):
    n, steps = 3000, 8
    p0 = (np.random.default_rng(4).standard_normal(n) * 0.02).astype(np.float32)
    grads = _grads(n, steps, 5)
    p = p0.copy()
    m = np.zeros(n, np.float32)
    for t, g in enumerate(grads, 1):
        oracle_mod.step_tensor("momentum", p, g, m, None, None, None, None, None, 2048, step=t,
                               lr=1e-2, beta1=0.9, beta2=0.0, eps=0.0, weight_decay=wd)
    pt, st = _torch_run(torch.optim.SGD, p0, grads, lr=_f(1e-2), momentum=_f(0.9), weight_decay=_f(wd),
                        foreach=False)
    _close(p, pt, np.abs(p0) + 1e-2 * np.abs(st["momentum_buffer"].numpy()).max() * steps, rtol=1e-6)
    _close(m, st["momentum_buffer"].numpy(), np.max(np.abs(m)), rtol=1e-5)


def test_momentum_first_step(oracle_mod):
    """P6: from zero state, momentum SGD's first step is p - lr * g, to one rounding."""
    n = 1000
    p0 = np.linspace(-1, 1, n).astype(np.float32)
    g = np.linspace(2, -3, n).astype(np.float32)
    p = p0.copy()
    m = np.zeros(n, np.float32)
    oracle_mod.step_tensor("momentum", p, g, m, None, None, None, None, None, 256, step=1,
                           lr=0.5, beta1=0.9, beta2=0.0, eps=0.0, weight_decay=0.0)
    np.testing.assert_array_equal(m, g)
    np.testing.assert_array_equal(p, (p0 - np.float32(0.5) * g).astype(np.float32))


def test_lion_sign_update(oracle_mod):
    """P6: Lion moves each parameter by exactly -lr*sign(b1*m + (1-b1)*g) after the decay, and
    the state becomes the b2-smoothed gradient."""
    n, lr, wd = 4000, 1e-4, 0.1
    rng = np.random.default_rng(6)
    p0 = (rng.standard_normal(n) * 0.02).astype(np.float32)
    m0 = (rng.standard_normal(n) * 1e-3).astype(np.float32)
    g = (rng.standard_normal(n) * 1e-3).astype(np.float32)
    g[:10] = 0.0
    m0[:10] = 0.0  # c == 0 -> no move
    p, m = p0.copy(), m0.copy()
    oracle_mod.step_tensor("lion", p, g, m, None, None, None, None, None, 2048, step=3,
                           lr=lr, beta1=0.9, beta2=0.99, eps=0.0, weight_decay=wd)
    decayed = (p0 * np.float32(1 - _f(lr) * _f(wd))).astype(np.float32)
    step = (decayed.astype(np.float64) - p) / _f(lr)
    c64 = _f(0.9) * m0.astype(np.float64) + (1 - _f(0.9)) * g
    clear = np.abs(c64) > 1e-9
    np.testing.assert_allclose(step[clear], np.sign(c64[clear]), atol=1e-3)
    assert np.all(p[:10] == decayed[:10])
    m64 = _f(0.99) * m0.astype(np.float64) + (1 - _f(0.99)) * g
    np.testing.assert_allclose(m, m64, rtol=1e-6, atol=1e-12)


def test_lion_decay_uses_the_old_parameter(oracle_mod):
    """Lion as X. Chen et al., "Symbolic Discovery of Optimization Algorithms", Algorithm 2:
    theta <- theta - lr * (sign(c) + wd * theta), the decay taken on the parameter before the
    sign step.  With lr * wd = 0.1 a decay applied after the sign step would be off by
    lr^2 * wd = 0.01 per element."""
    n, lr, wd = 5000, 0.1, 1.0
    rng = np.random.default_rng(16)
    p0 = rng.standard_normal(n).astype(np.float32)
    m0 = rng.standard_normal(n).astype(np.float32)
    g = rng.standard_normal(n).astype(np.float32)
    p, m = p0.copy(), m0.copy()
    oracle_mod.step_tensor("lion", p, g, m, None, None, None, None, None, 2048, step=1,
                           lr=lr, beta1=0.9, beta2=0.99, eps=0.0, weight_decay=wd)
    c64 = _f(0.9) * m0.astype(np.float64) + (1 - _f(0.9)) * g
    clear = np.abs(c64) > 1e-6
    assert clear.mean() > 0.99
    want = p0.astype(np.float64) - _f(lr) * (np.sign(c64) + _f(wd) * p0.astype(np.float64))
    err = np.abs(p[clear] - want[clear])
    assert np.all(err <= 4e-6 * (1 + np.abs(want[clear]))), err.max()


@pytest.mark.parametrize("wd", [0.0, 1e-2])
def test_rmsprop_matches_torch(oracle_mod, wd):
    """RMSprop (named by the page "bitsandbytes深度解析", section "优化器模块深度分析", as
    RMSprop8bit) against torch.optim.RMSprop in float64: alpha in beta1, eps outside the root,
    L2 weight decay, no momentum."""
    n, steps, alpha = 3000, 8, 0.99
    p0 = (np.random.default_rng(10).standard_normal(n) * 0.02).astype(np.float32)
    grads = _grads(n, steps, 11)
    p = p0.copy()
    v = np.zeros(n, np.float32)
    for t, g in enumerate(grads, 1):
        oracle_mod.step_tensor("rmsprop", p, g, v, None, None, None, None, None, 2048, step=t,
                               lr=1e-3, beta1=alpha, beta2=0.0, eps=1e-8, weight_decay=wd)
    pt, st = _torch_run(torch.optim.RMSprop, p0, grads, lr=_f(1e-3), alpha=_f(alpha), eps=_f(1e-8),
                        weight_decay=_f(wd), foreach=False)
    # each step moves p by about lr/sqrt(1-alpha) = 10 lr at most
    _close(p, pt, np.abs(p0) + 1e-2 * steps, rtol=1e-6)
    _close(v, st["square_avg"].numpy(), np.max(v), rtol=2e-5)


def test_rmsprop_first_step_closed_form(oracle_mod):
    """P5-style closed form: from zero state v' = (1-alpha) g^2, so step 1 is
    p - lr * g / (sqrt(1-alpha) |g| + eps)."""
    n, alpha, lr, eps = 4096, 0.9, 1e-3, 1e-8
    rng = np.random.default_rng(12)
    p0 = (rng.standard_normal(n) * 0.02).astype(np.float32)
    g = (rng.standard_normal(n) * 1e-3).astype(np.float32)
    p, v = p0.copy(), np.zeros(n, np.float32)
    oracle_mod.step_tensor("rmsprop", p, g, v, None, None, None, None, None, 256, step=1,
                           lr=lr, beta1=alpha, beta2=0.0, eps=eps, weight_decay=0.0)
    g64 = g.astype(np.float64)
    oma = 1 - _f(alpha)
    want = p0 - _f(lr) * g64 / (np.sqrt(oma) * np.abs(g64) + _f(eps))
    _close(p, want, np.abs(p0) + 10 * lr, rtol=0)
    _close(v, oma * g64 * g64, np.max(v), rtol=2e-6)


def test_rmsprop_8bit_step_matches_torch(oracle_mod):
    """8-bit RMSprop keeps its one state with the unsigned code: a step from a random 8-bit state
    equals torch's RMSprop from the dequantized state, and the new state is the nearest code."""
    n, B, alpha = 8192 + 5, 2048, 0.99
    rng = np.random.default_rng(13)
    code = oracle_mod.code_dynamic_unsigned()
    nb = (n + B - 1) // B
    p0 = (rng.standard_normal(n) * 0.02).astype(np.float32)
    g = (rng.standard_normal(n) * 1e-3).astype(np.float32)
    q = rng.integers(0, 256, n).astype(np.uint8)
    a = rng.uniform(1e-8, 1e-6, nb).astype(np.float32)
    v0 = _dequant(code, q, a, n, B)
    p = p0.copy()
    oracle_mod.step_tensor("rmsprop", p, g, q, None, a, None, code, None, B, step=4,
                           lr=1e-3, beta1=alpha, beta2=0.0, eps=1e-8, weight_decay=0.0)
    tp = torch.nn.Parameter(torch.from_numpy(p0.astype(np.float64)))
    opt = torch.optim.RMSprop([tp], lr=_f(1e-3), alpha=_f(alpha), eps=_f(1e-8), foreach=False)
    opt.state[tp] = {"step": torch.tensor(3.0), "square_avg": torch.from_numpy(v0.copy())}
    tp.grad = torch.from_numpy(g.astype(np.float64))
    opt.step()
    _close(p, tp.detach().numpy(), np.abs(p0) + 1e-2, rtol=1e-6)
    v1 = opt.state[tp]["square_avg"].numpy()
    want_a = np.array([np.max(v1[i:i + B]) for i in range(0, n, B)])
    np.testing.assert_allclose(a, want_a, rtol=1e-6)
    xn = v1 / np.repeat(want_a, B)[:n]
    qq, margin = _nearest_exact(code, xn)
    far = margin > 1e-5 * np.maximum(np.abs(xn), 1e-7)
    assert far.mean() > 0.99
    np.testing.assert_array_equal(q[far], qq[far])


# ----------------------------------------------------------------------- 8-bit state path
def _dequant(code, q, absmax, n, B):
    return code[q].astype(np.float64) * np.repeat(absmax.astype(np.float64), B)[:n]


def _nearest_exact(code, xn):
    c64 = code.astype(np.float64)
    hi = np.clip(np.searchsorted(c64, xn, side="left"), 1, len(code) - 1)
    lo = hi - 1
    return np.where(c64[hi] - xn < xn - c64[lo], hi, lo), np.minimum(c64[hi] - xn, xn - c64[lo])


def test_8bit_first_step_equals_32bit(oracle_mod):
    """From zero state the dequantized state is exactly zero, so the 8-bit and 32-bit paths give
    bit-identical parameters at step 1; the stored 8-bit state is the nearest code of m/absmax."""
    n, B = 65536 + 333, 2048
    rng = np.random.default_rng(8)
    p0 = (rng.standard_normal(n) * 0.02).astype(np.float32)
    g = (rng.standard_normal(n) * 1e-3).astype(np.float32)
    c1, c2 = oracle_mod.code_dynamic_signed(), oracle_mod.code_dynamic_unsigned()
    nb = (n + B - 1) // B
    p8 = p0.copy()
    q1 = np.full(n, 127, np.uint8)
    q2 = np.zeros(n, np.uint8)
    a1 = np.zeros(nb, np.float32)
    a2 = np.zeros(nb, np.float32)
    oracle_mod.step_tensor("adamw", p8, g, q1, q2, a1, a2, c1, c2, B, step=1, **HP)
    p32 = p0.copy()
    m = np.zeros(n, np.float32)
    v = np.zeros(n, np.float32)
    oracle_mod.step_tensor("adamw", p32, g, m, v, None, None, None, None, B, step=1, **HP)
    np.testing.assert_array_equal(p8, p32)
    # requantized state: block absmax of the 32-bit state, then the nearest code
    for a, q, s, code in ((a1, q1, m, c1), (a2, q2, v, c2)):
        want_a = np.array([np.max(np.abs(s[i:i + B])) for i in range(0, n, B)], np.float32)
        np.testing.assert_array_equal(a, want_a)
        xn = (s / np.repeat(want_a, B)[:n]).astype(np.float32).astype(np.float64)
        qq, _ = _nearest_exact(code, xn)
        np.testing.assert_array_equal(q, qq)


def test_8bit_step_from_quantized_state_matches_torch(oracle_mod):
    """A step from a random 8-bit state equals torch's AdamW run from the dequantized state; the
    new state is the nearest code of the new moments (checked away from decision boundaries)."""
    n, B, t = 8192 + 77, 2048, 7
    rng = np.random.default_rng(9)
    c1, c2 = oracle_mod.code_dynamic_signed(), oracle_mod.code_dynamic_unsigned()
    nb = (n + B - 1) // B
    p0 = (rng.standard_normal(n) * 0.02).astype(np.float32)
    g = (rng.standard_normal(n) * 1e-3).astype(np.float32)
    q1 = rng.integers(0, 256, n).astype(np.uint8)
    q2 = rng.integers(0, 256, n).astype(np.uint8)
    a1 = rng.uniform(1e-4, 1e-3, nb).astype(np.float32)
    a2 = rng.uniform(1e-8, 1e-6, nb).astype(np.float32)
    m0 = _dequant(c1, q1, a1, n, B)
    v0 = _dequant(c2, q2, a2, n, B)
    p = p0.copy()
    oracle_mod.step_tensor("adamw", p, g, q1, q2, a1, a2, c1, c2, B, step=t, **HP)

    tp = torch.nn.Parameter(torch.from_numpy(p0.astype(np.float64)))
    opt = torch.optim.AdamW([tp], lr=_f(1e-3), betas=(_f(0.9), _f(0.999)), eps=_f(1e-8),
                            weight_decay=_f(0.01), foreach=False)
    opt.state[tp] = {"step": torch.tensor(float(t - 1)), "exp_avg": torch.from_numpy(m0.copy()),
                     "exp_avg_sq": torch.from_numpy(v0.copy())}
    tp.grad = torch.from_numpy(g.astype(np.float64))
    opt.step()
    _close(p, tp.detach().numpy(), np.abs(p0) + 1e-3, rtol=1e-6)
    m1 = opt.state[tp]["exp_avg"].numpy()
    v1 = opt.state[tp]["exp_avg_sq"].numpy()
    for a, q, s, code in ((a1, q1, m1, c1), (a2, q2, v1, c2)):
        want_a = np.array([np.max(np.abs(s[i:i + B])) for i in range(0, n, B)])
        np.testing.assert_allclose(a, want_a, rtol=1e-6)
        xn = s / np.repeat(want_a, B)[:n]
        qq, margin = _nearest_exact(code, xn)
        far = margin > 1e-5 * np.maximum(np.abs(xn), 1e-7)  # not near a decision boundary
        assert far.mean() > 0.99
        np.testing.assert_array_equal(q[far], qq[far])


def test_zero_gradient_zero_state_stays(oracle_mod):
    """P6: zero gradient on zero 8-bit state keeps code(0) and absmax 0."""
    n, B = 5000, 2048
    c1, c2 = oracle_mod.code_dynamic_signed(), oracle_mod.code_dynamic_unsigned()
    nb = (n + B - 1) // B
    p = np.ones(n, np.float32)
    q1 = np.full(n, 127, np.uint8)
    q2 = np.zeros(n, np.uint8)
    a1 = np.zeros(nb, np.float32)
    a2 = np.zeros(nb, np.float32)
    oracle_mod.step_tensor("adamw", p, np.zeros(n, np.float32), q1, q2, a1, a2, c1, c2, B, step=1,
                           lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.0)
    assert np.all(q1 == 127) and np.all(q2 == 0) and np.all(a1 == 0) and np.all(a2 == 0)
    assert np.all(p == 1.0)


def test_state_bytes_per_param():
    """P8: 8-bit Adam keeps two one-byte codes per parameter (2 B/param of state, vs 8 B for two
    fp32 moments: the 75% reduction of the bitsandbytes skill page, Workflow 3), plus one fp32
    absmax per block per state."""
    n, B = 7_000_000_000, 2048
    state8 = 2 * n + 2 * 4 * ((n + B - 1) // B)
    state32 = 8 * n
    assert abs(state8 / n - 2.0) < 0.01
    assert abs(1 - state8 / state32 - 0.75) < 0.002


def test_bf16_gradients_are_widened_exactly(oracle_mod):
    n = 3000
    rng = np.random.default_rng(11)
    p0 = (rng.standard_normal(n) * 0.02).astype(np.float32)
    gt = torch.from_numpy((rng.standard_normal(n) * 1e-3).astype(np.float32)).to(torch.bfloat16)
    bits = gt.view(torch.int16).numpy().view(np.uint16)
    outs = []
    for g in (bits, gt.float().numpy()):
        p = p0.copy()
        m = np.zeros(n, np.float32)
        v = np.zeros(n, np.float32)
        oracle_mod.step_tensor("adamw", p, g, m, v, None, None, None, None, 2048, step=1, **HP)
        outs.append(p)
    np.testing.assert_array_equal(outs[0], outs[1])


_TORCH_OPT = {"adamw": "AdamW", "adam": "Adam", "momentum": "SGD", "rmsprop": "RMSprop"}


@settings(max_examples=60, deadline=None)
@given(optim=st.sampled_from(sorted(_TORCH_OPT)), n=st.integers(1, 600), steps=st.integers(1, 6),
       lr=st.floats(1e-5, 1e-2), b1=st.floats(0.5, 0.99), b2=st.floats(0.9, 0.9999),
       eps=st.sampled_from([1e-10, 1e-8, 1e-6]), wd=st.sampled_from([0.0, 1e-3, 0.1]), seed=st.integers(0, 2**31))
def test_32bit_step_matches_torch_random_hyperparameters(oracle_mod, optim, n, steps, lr, b1, b2, eps, wd, seed):
    """Random hyper-parameters, lengths and step counts: the 32-bit oracle step tracks
    torch.optim (float64) for AdamW, Adam (L2), SGD with momentum and RMSprop (alpha = beta1)."""
    p0 = (np.random.default_rng(seed).standard_normal(n) * 0.02).astype(np.float32)
    grads = _grads(n, steps, seed + 1)
    p = p0.copy()
    m = np.zeros(n, np.float32)
    v = np.zeros(n, np.float32) if optim in ("adamw", "adam") else None
    for t, g in enumerate(grads, 1):
        oracle_mod.step_tensor(optim, p, g, m, v, None, None, None, None, 256, step=t,
                               lr=lr, beta1=b1, beta2=b2 if v is not None else 0.0, eps=eps, weight_decay=wd)
    kw = dict(lr=_f(lr), weight_decay=_f(wd), foreach=False)
    if optim in ("adamw", "adam"):
        kw.update(betas=(_f(b1), _f(b2)), eps=_f(eps))
    elif optim == "momentum":
        kw.update(momentum=_f(b1))
    else:
        kw.update(alpha=_f(b1), eps=_f(eps))
    pt, st_ = _torch_run(getattr(torch.optim, _TORCH_OPT[optim]), p0, grads, **kw)
    _close(p, pt, np.abs(p0) + np.abs(pt - p0) + lr * steps, rtol=4e-6, ulps=8)
    first = {"adamw": "exp_avg", "adam": "exp_avg", "momentum": "momentum_buffer", "rmsprop": "square_avg"}[optim]
    _close(m, st_[first].numpy(), np.max(np.abs(m)), rtol=5e-5)
    if v is not None:
        _close(v, st_["exp_avg_sq"].numpy(), np.max(v), rtol=5e-5)


@settings(max_examples=50, deadline=None)
@given(optim=st.sampled_from(sorted(_TORCH_OPT)), n=st.integers(1, 5000), B=st.sampled_from([256, 2048]),
       t=st.integers(1, 30), lr=st.floats(1e-5, 1e-2), b1=st.floats(0.5, 0.99), b2=st.floats(0.9, 0.9999),
       wd=st.sampled_from([0.0, 0.01]), seed=st.integers(0, 2**31))
def test_8bit_step_random_state_matches_torch(oracle_mod, optim, n, B, t, lr, b1, b2, wd, seed):
    """Random 8-bit states, scales, hyper-parameters and lengths: the step equals torch.optim run
    from the dequantized state, each new block scale is the block's largest new |state|, and
    each new code is the exact nearest code of state / scale wherever that quotient is not
    within a relative 1e-5 of a decision midpoint."""
    rng = np.random.default_rng(seed)
    two = optim in ("adamw", "adam")
    c1 = oracle_mod.code_dynamic_unsigned() if optim == "rmsprop" else oracle_mod.code_dynamic_signed()
    c2 = oracle_mod.code_dynamic_unsigned()
    nb = (n + B - 1) // B
    p0 = (rng.standard_normal(n) * 0.02).astype(np.float32)
    g = (rng.standard_normal(n) * 1e-3).astype(np.float32)
    q1 = rng.integers(0, 256, n).astype(np.uint8)
    q2 = rng.integers(0, 256, n).astype(np.uint8)
    a1 = rng.uniform(1e-8, 1e-6, nb).astype(np.float32) if optim == "rmsprop" else \
        rng.uniform(1e-4, 1e-3, nb).astype(np.float32)
    a2 = rng.uniform(1e-8, 1e-6, nb).astype(np.float32)
    m0 = (c1[q1] * np.repeat(a1, B)[:n]).astype(np.float32)  # the dequantized state, binary32
    v0 = (c2[q2] * np.repeat(a2, B)[:n]).astype(np.float32)
    p = p0.copy()
    oracle_mod.step_tensor(optim, p, g, q1, q2 if two else None, a1, a2 if two else None, c1, c2 if two else None,
                           B, step=t, lr=lr, beta1=b1, beta2=b2 if two else 0.0, eps=1e-8, weight_decay=wd)

    tp = torch.nn.Parameter(torch.from_numpy(p0.astype(np.float64)))
    kw = dict(lr=_f(lr), weight_decay=_f(wd), foreach=False)
    m64 = torch.from_numpy(m0.astype(np.float64))
    if two:
        kw.update(betas=(_f(b1), _f(b2)), eps=_f(1e-8))
        state = {"step": torch.tensor(float(t - 1)), "exp_avg": m64, "exp_avg_sq": torch.from_numpy(v0.astype(np.float64))}
    elif optim == "momentum":
        kw.update(momentum=_f(b1))
        state = {"momentum_buffer": m64}
    else:
        kw.update(alpha=_f(b1), eps=_f(1e-8))
        state = {"step": torch.tensor(float(t - 1)), "square_avg": m64}
    opt = getattr(torch.optim, _TORCH_OPT[optim])([tp], **kw)
    opt.state[tp] = state
    tp.grad = torch.from_numpy(g.astype(np.float64))
    opt.step()
    pt = tp.detach().numpy()
    _close(p, pt, np.abs(p0) + np.abs(pt - p0) + lr, rtol=4e-6, ulps=8)

    first = {"adamw": "exp_avg", "adam": "exp_avg", "momentum": "momentum_buffer", "rmsprop": "square_avg"}[optim]
    checks = [(a1, q1, opt.state[tp][first].numpy(), c1)]
    if two:
        checks.append((a2, q2, opt.state[tp]["exp_avg_sq"].numpy(), c2))
    for a, q, s, code in checks:
        want_a = np.array([np.max(np.abs(s[i:i + B])) for i in range(0, n, B)])
        np.testing.assert_allclose(a, want_a, rtol=2e-5)
        xn = s / np.repeat(want_a, B)[:n]
        mids = (code[:-1].astype(np.float64) + code[1:].astype(np.float64)) / 2
        k = np.clip(np.searchsorted(mids, xn), 1, mids.size - 1)
        gap = np.minimum(np.abs(xn - mids[k - 1]), np.abs(xn - mids[np.minimum(k, mids.size - 1)]))
        far = gap > 1e-5 * np.maximum(np.abs(xn), 1e-7)
        qq, _ = _nearest_exact(code, xn)
        np.testing.assert_array_equal(q[far], qq[far])
        if n >= 1000:
            assert far.mean() > 0.95


@settings(max_examples=60, deadline=None)
@given(optim=st.sampled_from(["adamw", "adam", "lion", "momentum", "rmsprop"]), n=st.integers(1, 9000),
       B=st.sampled_from([256, 2048]), split=st.floats(0, 1), t=st.integers(1, 9), seed=st.integers(0, 2**31))
def test_blocks_are_independent(oracle_mod, optim, n, B, split, t, seed):
    """Blocks are quantized and stepped independently (abstract of "8-bit Optimizers via
    Block-wise Quantization"): stepping the block range in two parts, at any split, gives exactly
    the result of one call over all blocks."""
    rng = np.random.default_rng(seed)
    two = optim in ("adamw", "adam")
    c1 = oracle_mod.code_dynamic_unsigned() if optim == "rmsprop" else oracle_mod.code_dynamic_signed()
    c2 = oracle_mod.code_dynamic_unsigned()
    nb = (n + B - 1) // B
    k = int(round(split * nb))
    base = dict(p=(rng.standard_normal(n) * 0.02).astype(np.float32),
                g=(rng.standard_normal(n) * 1e-3).astype(np.float32),
                q1=rng.integers(0, 256, n).astype(np.uint8), q2=rng.integers(0, 256, n).astype(np.uint8),
                a1=rng.uniform(1e-8, 1e-3, nb).astype(np.float32), a2=rng.uniform(1e-8, 1e-6, nb).astype(np.float32))
    hp = dict(lr=1e-3, beta1=0.9, beta2=0.999 if two else 0.0, eps=1e-8, weight_decay=0.01)
    runs = []
    for ranges in ([(0, nb)], [(0, k), (k, nb)]):
        d = {key: v.copy() for key, v in base.items()}
        for r in ranges:
            oracle_mod.step_tensor(optim, d["p"], d["g"], d["q1"], d["q2"] if two else None, d["a1"],
                                   d["a2"] if two else None, c1, c2 if two else None, B, step=t, block_range=r, **hp)
        runs.append(d)
    for key in base:
        np.testing.assert_array_equal(runs[0][key], runs[1][key])
