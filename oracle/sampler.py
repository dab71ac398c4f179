"""Canvas sampler and adaptive stop rule (oracle side).

What one denoise step's sampler computes, per canvas position i with logits
x_i over the vocabulary (temperature 1):

    p_i     = softmax(x_i)                       (float64)
    conf_i  = max_v p_i[v]                       confidence of the best token
    H_i     = -sum_v p_i[v] ln p_i[v]            entropy in nats (0 ln 0 = 0)
    a_i     = smallest v with x_i[v] = max x_i   argmax, lowest index on ties
    next_i  = a_i                 if conf_i >= tau        (lock, [course] 2.1,
              uniform id(seed, block, t, i)   otherwise    re-noise, [canvas] step 3,
                                                           [uniform])

Locks are stateless: a position locked at step t is re-decided at step t+1 from
that step's logits, which is what lets a confident token later be re-noised
when its confidence drops ([uniform]).

Stop rule ([canvas] step 3): steps are numbered t = 1, 2, ...; after step t the
block stops if t >= 2, the mean entropy over all canvas positions is below the
bound (0.005), and the argmax vector equals the previous step's argmax vector
element for element.  If no step meets this, the block stops at the step cap
(48).  In fixed-step mode exactly `fixed_steps` steps run and the step at which
the rule would have stopped is still reported.  The committed block is the
argmax vector of the stop step ([canvas] step 4).
"""
import numpy as np

from .philox import TAG_INIT, TAG_RENOISE, uniform_ids

TAU = 0.9
H_BOUND = 0.005
MAX_STEPS = 48


def row_stats(logits):
    """Per-row (conf, entropy in nats, argmax) of logits [T, V], all from float64 softmax."""
    x = np.asarray(logits, dtype=np.float64)
    if x.ndim != 2 or x.shape[1] == 0:
        raise ValueError("logits must be [T, V] with V >= 1")
    m = x.max(axis=1, keepdims=True)
    e = np.exp(x - m)
    s = e.sum(axis=1, keepdims=True)
    p = e / s
    conf = p.max(axis=1)
    with np.errstate(divide="ignore", invalid="ignore"):
        plogp = np.where(p > 0.0, p * np.log(np.where(p > 0.0, p, 1.0)), 0.0)
    ent = -plogp.sum(axis=1)
    amax = np.argmax(x, axis=1)  # numpy returns the first (lowest) index among equal maxima
    return conf, ent, amax.astype(np.int64)


def canvas_init(seed, block, canvas_len, vocab):
    """Initial canvas: ids uniform over the whole vocabulary ([canvas] step 2)."""
    return uniform_ids(seed, block, 0, np.arange(canvas_len), TAG_INIT, vocab)


def sample_update(conf, amax, seed, block, step, vocab, tau=TAU):
    """Next canvas: lock confident positions to their argmax, re-noise the rest."""
    conf = np.asarray(conf, dtype=np.float64)
    pos = np.arange(conf.shape[0])
    noise = uniform_ids(seed, block, step, pos, TAG_RENOISE, vocab)
    return np.where(conf >= tau, np.asarray(amax, dtype=np.int64), noise), conf >= tau


def would_stop(step, mean_entropy, amax, prev_amax, h_bound=H_BOUND):
    """The two-condition stop test after step `step` (1-based)."""
    if step < 2 or prev_amax is None:
        return False
    return bool(mean_entropy < h_bound) and bool(np.array_equal(amax, prev_amax))


def run_block(logits_for_step, seed, block, vocab, canvas_len, *, max_steps=MAX_STEPS,
              fixed_steps=None, tau=TAU, h_bound=H_BOUND):
    """Drive one block given a callback logits_for_step(t, canvas) -> logits [T, V].

    Returns a dict: committed ids, stop step (steps actually run), would-stop step
    (first step meeting the rule, or None), and per-step records of canvas, argmax,
    conf, entropy and mean entropy.
    """
    canvas = canvas_init(seed, block, canvas_len, vocab)
    n_steps = fixed_steps if fixed_steps is not None else max_steps
    prev = None
    first_stop = None
    steps = []
    stop_step = n_steps
    for t in range(1, n_steps + 1):
        logits = logits_for_step(t, canvas)
        conf, ent, amax = row_stats(logits)
        hbar = float(ent.mean())
        stop_now = would_stop(t, hbar, amax, prev, h_bound)
        nxt, locked = sample_update(conf, amax, seed, block, t, vocab, tau)
        steps.append(dict(step=t, canvas_in=canvas, amax=amax, conf=conf, entropy=ent,
                          mean_entropy=hbar, locked=locked, canvas_out=nxt, stop=stop_now))
        if stop_now and first_stop is None:
            first_stop = t
        canvas = nxt
        prev = amax
        if stop_now and fixed_steps is None:
            stop_step = t
            break
    committed = steps[stop_step - 1]["amax"]
    return dict(committed=committed, stop_step=stop_step, would_stop_step=first_stop, steps=steps,
                canvas=canvas)
