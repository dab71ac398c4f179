"""Pins for the oracle's sampler statistics, lock/re-noise and stop rule.

The stop-rule sequences are built so that the stop step is known from their
construction alone (closed-form binary entropies), not from the oracle.
"""
import math

import numpy as np
import pytest
from scipy import special

from oracle import sampler as smp
from oracle.philox import philox4x32_10, uniform_ids


@pytest.mark.parametrize("vocab", [2, 3, 4, 8, 1000])
def test_stats_against_scipy(vocab):
    rng = np.random.default_rng(vocab)
    x = rng.standard_normal((64, vocab)) * rng.uniform(0.1, 20, (64, 1))
    conf, ent, amax = smp.row_stats(x)
    p = special.softmax(x, axis=1)
    assert np.allclose(ent, special.entr(p).sum(axis=1), rtol=0, atol=1e-12)
    assert np.allclose(conf, p.max(axis=1), rtol=1e-13, atol=0)
    # a different route to the same entropy: H = logsumexp(x) - E_p[x]
    assert np.allclose(ent, special.logsumexp(x, axis=1) - (p * x).sum(axis=1), atol=1e-9)
    assert np.array_equal(amax, np.argmax(x, axis=1))


def test_closed_forms():
    v = 16
    conf, ent, amax = smp.row_stats(np.full((1, v), 3.25))
    assert math.isclose(ent[0], math.log(v), rel_tol=1e-14) and math.isclose(conf[0], 1 / v, rel_tol=1e-14)
    assert amax[0] == 0
    # two equal maxima, the rest effectively -inf: entropy ln 2, argmax the lower index
    x = np.full((1, v), -1e30)
    x[0, 5] = x[0, 11] = 2.0
    conf, ent, amax = smp.row_stats(x)
    assert math.isclose(ent[0], math.log(2), rel_tol=1e-14) and amax[0] == 5 and math.isclose(conf[0], 0.5)
    # one overwhelming logit: entropy 0, confidence 1
    x = np.zeros((1, v))
    x[0, 9] = 1e4
    conf, ent, amax = smp.row_stats(x)
    assert ent[0] == 0.0 and conf[0] == 1.0 and amax[0] == 9
    # V = 2: binary entropy of sigmoid(c)
    c = 1.7
    conf, ent, _ = smp.row_stats(np.array([[c, 0.0]]))
    p = 1 / (1 + math.exp(-c))
    assert math.isclose(ent[0], -p * math.log(p) - (1 - p) * math.log(1 - p), rel_tol=1e-13)
    assert math.isclose(conf[0], p, rel_tol=1e-14)


def test_lock_and_renoise_hand_worked():
    # V = 8: row 0 conf = e^10/(e^10+7) > 0.9 locks to 0; row 1 uniform (conf 1/8) is re-noised;
    # row 2 conf = 9*7/(9*7+7) = 0.9 exactly in real arithmetic, row 3 just below (0.8).
    v = 8
    x = np.zeros((4, v))
    x[0, 0] = 10.0
    x[2, 6] = math.log(63.0)
    x[3, 3] = math.log(28.0)
    conf, _, amax = smp.row_stats(x)
    assert conf[0] > 0.9 and abs(conf[1] - 0.125) < 1e-15 and abs(conf[2] - 0.9) < 1e-15
    assert abs(conf[3] - 0.8) < 1e-15
    seed, block, step = 0xDEADBEEF_00000007, 2, 5
    nxt, locked = smp.sample_update(conf, amax, seed, block, step, v)
    r0 = philox4x32_10(np.arange(4), step, block, 1, seed & 0xFFFFFFFF, seed >> 32)[0]
    draw = (r0 * np.uint64(v)) >> np.uint64(32)
    assert nxt[0] == 0 and locked[0]
    assert nxt[1] == int(draw[1]) and not locked[1]
    assert nxt[3] == int(draw[3]) and not locked[3]
    # row 2 sits on the threshold: the lock is inclusive, so it locks iff conf >= 0.9 in float64
    assert locked[2] == (conf[2] >= 0.9)
    assert nxt[2] == (6 if conf[2] >= 0.9 else int(draw[2]))
    # tau above 1 never locks; tau 0 always locks
    nxt_none, lk = smp.sample_update(conf, amax, seed, block, step, v, tau=1.5)
    assert not lk.any() and np.array_equal(nxt_none, draw.astype(np.int64))
    nxt_all, lk = smp.sample_update(conf, amax, seed, block, step, v, tau=0.0)
    assert lk.all() and np.array_equal(nxt_all, amax)


def test_canvas_init_is_tag0_step0():
    ids = smp.canvas_init(11, 3, 256, 1 << 18)
    assert np.array_equal(ids, uniform_ids(11, 3, 0, np.arange(256), 0, 1 << 18))


def _binary_rows(c_of_t, argmax_of_t, rows=4):
    """Logits [rows, 2]: winner logit 0, loser -c; entropy is the binary entropy of sigmoid(-c)."""
    def f(t, canvas):
        x = np.zeros((rows, 2))
        a = argmax_of_t(t)
        x[:, 1 - a] = -c_of_t(t)
        return x
    return f


def _hb(c):
    p = 1 / (1 + math.exp(c))
    return -p * math.log(p) - (1 - p) * math.log(1 - p)


def test_binary_entropy_levels():
    # the two levels used below sit well on either side of the 0.005 bound
    assert _hb(5.0) > 0.02 and _hb(10.0) < 0.001


@pytest.mark.parametrize("t_star", [2, 7, 20, 48])
def test_stop_entropy_gated(t_star):
    f = _binary_rows(lambda t: 10.0 if t >= t_star else 5.0, lambda t: 0)
    res = smp.run_block(f, 1, 0, 2, 4)
    assert res["stop_step"] == t_star and res["would_stop_step"] == t_star
    assert np.array_equal(res["committed"], np.zeros(4, np.int64))


@pytest.mark.parametrize("t_star", [3, 9])
def test_stop_argmax_gated(t_star):
    # entropy is low from step 1, but the argmax alternates until step t_star, then holds:
    # the first step whose argmax equals the previous one is t_star + 1.
    f = _binary_rows(lambda t: 10.0, lambda t: (t % 2) if t <= t_star else (t_star % 2))
    res = smp.run_block(f, 1, 0, 2, 4)
    assert res["stop_step"] == t_star + 1
    assert np.array_equal(res["committed"], np.full(4, t_star % 2))


def test_never_converges_hits_cap():
    f = _binary_rows(lambda t: 5.0, lambda t: 0)
    res = smp.run_block(f, 1, 0, 2, 4)
    assert res["stop_step"] == 48 and res["would_stop_step"] is None and len(res["steps"]) == 48


def test_step_one_never_stops():
    f = _binary_rows(lambda t: 10.0, lambda t: 0)
    res = smp.run_block(f, 1, 0, 2, 4)
    assert res["stop_step"] == 2


def test_fixed_mode_runs_all_steps_and_reports_would_stop():
    f = _binary_rows(lambda t: 10.0 if t >= 6 else 5.0, lambda t: 0 if t < 12 else 1)
    res = smp.run_block(f, 1, 0, 2, 4, fixed_steps=16)
    assert res["stop_step"] == 16 and res["would_stop_step"] == 6 and len(res["steps"]) == 16
    assert np.array_equal(res["committed"], np.ones(4, np.int64))


def test_mean_entropy_includes_every_position():
    # one uncertain row keeps the mean above the bound even if the others are certain
    def f(t, canvas):
        x = np.zeros((4, 2))
        x[:3, 1] = -30.0
        return x
    res = smp.run_block(f, 1, 0, 2, 4)
    assert res["stop_step"] == 48
    assert math.isclose(res["steps"][0]["mean_entropy"], (math.log(2) + 3 * _hb(30.0)) / 4, rel_tol=1e-12)


# ---- sampler variants: temperature, entropy-bound locking, sticky locks ------------------------

@pytest.mark.parametrize("vocab,temp", [(2, 0.3), (5, 2.5), (1000, 0.7), (1000, 4.0)])
def test_temperature_stats_against_scipy(vocab, temp):
    from scipy.special import entr, softmax
    rng = np.random.default_rng(vocab)
    x = rng.standard_normal((16, vocab)) * 3
    conf, ent, amax = smp.row_stats(x, temperature=temp)
    p = softmax(x / temp, axis=1)
    assert np.allclose(conf, p.max(axis=1), rtol=1e-12, atol=1e-15)
    assert np.allclose(ent, entr(p).sum(axis=1), rtol=1e-10, atol=1e-13)
    assert np.array_equal(amax, np.argmax(x, axis=1))


def test_temperature_limits():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((8, 64))
    _, ent, _ = smp.row_stats(x, temperature=1e7)
    assert np.allclose(ent, np.log(64), atol=1e-6)  # hot: uniform over the vocabulary
    x[:, 7] = x.max(axis=1) + 0.5  # a unique maximum at index 7, 0.5 above the rest
    conf, ent, amax = smp.row_stats(x, temperature=1e-3)
    assert np.all(amax == 7) and np.all(conf >= 1 - 1e-15) and np.all(ent < 1e-100)
    with pytest.raises(ValueError):
        smp.row_stats(x, temperature=0.0)


def test_entropy_bound_rule_hand_worked():
    # row 0: one logit 20 above three others -> H ~ 3 * 21 e^-20 << 0.1: lock to 0
    # row 1: uniform over 4 -> H = ln 4 > 0.1: re-noise
    # row 2: two equal maxima -> H >= ln 2 > 0.1 although conf = 0.5: re-noise
    # row 3: conf 0.95 (locks under the confidence rule) but entropy above a bound of 0.1
    x = np.array([[20.0, 0, 0, 0], [1.0, 1, 1, 1], [3.0, 3, 0, 0],
                  [np.log(0.95 / 0.05 * 3), 0, 0, 0]])
    conf, ent, amax = smp.row_stats(x)
    assert ent[3] > 0.1 and conf[3] > 0.9
    nxt, lock = smp.sample_update(conf, amax, 9, 0, 1, 4, entropy=ent, rule="entropy_bound",
                                  entropy_bound=0.1)
    assert lock.tolist() == [True, False, False, False]
    noise = smp.uniform_ids(9, 0, 1, np.arange(4), smp.TAG_RENOISE, 4)
    assert nxt.tolist() == [0, noise[1], noise[2], noise[3]]
    _, lock_c = smp.sample_update(conf, amax, 9, 0, 1, 4)
    assert lock_c.tolist() == [True, False, False, True]
    with pytest.raises(ValueError):
        smp.sample_update(conf, amax, 9, 0, 1, 4, rule="entropy_bound")


def test_sticky_lock_keeps_its_token():
    v = 8
    conf1, amax1 = np.array([0.95, 0.2]), np.array([3, 1])
    nxt1, lock1 = smp.sample_update(conf1, amax1, 5, 0, 1, v)
    assert nxt1[0] == 3 and lock1.tolist() == [True, False]
    conf2, amax2 = np.array([0.3, 0.2]), np.array([6, 2])  # position 0 loses its confidence
    sticky, lock_s = smp.sample_update(conf2, amax2, 5, 0, 2, v, sticky=True, prev_canvas=nxt1,
                                       prev_locked=lock1)
    plain, lock_p = smp.sample_update(conf2, amax2, 5, 0, 2, v)
    noise2 = smp.uniform_ids(5, 0, 2, np.arange(2), smp.TAG_RENOISE, v)
    assert sticky.tolist() == [3, noise2[1]] and lock_s.tolist() == [True, False]
    assert plain.tolist() == [noise2[0], noise2[1]] and lock_p.tolist() == [False, False]


def test_sticky_block_commits_locked_tokens():
    # position 0 is confident on token 2 at step 1 only, then flat; position 1 is never confident
    v, steps = 4, 3

    def logits(t, canvas):
        x = np.zeros((2, v))
        if t == 1:
            x[0, 2] = 10.0
        else:
            x[0, 1] = 0.01  # argmax moves to 1, confidence ~ 0.25
        return x

    plain = smp.run_block(logits, 3, 0, v, 2, fixed_steps=steps)
    sticky = smp.run_block(logits, 3, 0, v, 2, fixed_steps=steps, sticky=True)
    assert plain["committed"].tolist() == [1, 0]        # argmax vector of the last step
    assert sticky["committed"].tolist() == [2, 0]       # the sticky lock keeps token 2
    assert sticky["steps"][2]["canvas_in"][0] == 2      # and feeds it to every later step
    assert plain["steps"][2]["canvas_in"][0] != 2 or plain["steps"][1]["canvas_out"][0] != 2
