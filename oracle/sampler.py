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

Variants (none is the default; the pages name them without defining them, so each is the
plainest reading):
  * temperature T > 0: every statistic above is taken from softmax(x_i / T); the argmax does not
    depend on T.  The pages fix temperature among the generation settings of an A/B test
    ([canvas], "同一條起跑線" list) without giving its role in the sampler.
  * rule "entropy_bound" (the vLLM recipe's `diffusion_sampler: entropy_bound`,
    `diffusion_entropy_bound: 0.1`, [canvas] A/B commands): position i locks when H_i <= bound
    instead of when conf_i >= tau.
  * sticky locks: a position that locked keeps its token for the rest of the block and is not
    re-decided (the default re-decides every step, as [uniform] describes).
The stop rule is unchanged and uses the (temperature-T) entropies.  The committed block takes a
locked position's canvas token and every other position's argmax; without sticky locks a locked
token is the argmax, so this is the argmax vector of the stop step.
"""
import numpy as np

from .philox import TAG_INIT, TAG_RENOISE, uniform_ids

TAU = 0.9
H_BOUND = 0.005
MAX_STEPS = 48


def row_stats(logits, temperature=1.0):
    """Per-row (conf, entropy in nats, argmax) of logits [T, V], all from float64 softmax of
    logits / temperature; the argmax is that of the logits themselves."""
    x = np.asarray(logits, dtype=np.float64)
    if x.ndim != 2 or x.shape[1] == 0:
        raise ValueError("logits must be [T, V] with V >= 1")
    if not temperature > 0:
        raise ValueError("temperature must be positive")
    amax = np.argmax(x, axis=1)  # numpy returns the first (lowest) index among equal maxima
    if temperature != 1.0:
        x = x / temperature
    m = x.max(axis=1, keepdims=True)
    e = np.exp(x - m)
    s = e.sum(axis=1, keepdims=True)
    p = e / s
    conf = p.max(axis=1)
    with np.errstate(divide="ignore", invalid="ignore"):
        plogp = np.where(p > 0.0, p * np.log(np.where(p > 0.0, p, 1.0)), 0.0)
    ent = -plogp.sum(axis=1)
    return conf, ent, amax.astype(np.int64)


def canvas_init(seed, block, canvas_len, vocab):
    """Initial canvas: ids uniform over the whole vocabulary ([canvas] step 2)."""
    return uniform_ids(seed, block, 0, np.arange(canvas_len), TAG_INIT, vocab)


def sample_update(conf, amax, seed, block, step, vocab, tau=TAU, *, entropy=None,
                  rule="confidence", entropy_bound=0.1, sticky=False, prev_canvas=None,
                  prev_locked=None):
    """Next canvas: lock confident positions to their argmax, re-noise the rest.

    rule "confidence" locks conf >= tau; rule "entropy_bound" locks entropy <= entropy_bound.
    sticky: positions in prev_locked keep their prev_canvas token and stay locked.
    Returns (next canvas, locked mask).
    """
    conf = np.asarray(conf, dtype=np.float64)
    pos = np.arange(conf.shape[0])
    noise = uniform_ids(seed, block, step, pos, TAG_RENOISE, vocab)
    if rule == "confidence":
        lock = conf >= tau
    elif rule == "entropy_bound":
        if entropy is None:
            raise ValueError("the entropy_bound rule needs the entropies")
        lock = np.asarray(entropy, dtype=np.float64) <= entropy_bound
    else:
        raise ValueError(f"unknown lock rule {rule!r}")
    nxt = np.where(lock, np.asarray(amax, dtype=np.int64), noise)
    if sticky and prev_locked is not None:
        kept = np.asarray(prev_locked, dtype=bool)
        nxt = np.where(kept, np.asarray(prev_canvas, dtype=np.int64), nxt)
        lock = lock | kept
    return nxt, lock


def would_stop(step, mean_entropy, amax, prev_amax, h_bound=H_BOUND):
    """The two-condition stop test after step `step` (1-based)."""
    if step < 2 or prev_amax is None:
        return False
    return bool(mean_entropy < h_bound) and bool(np.array_equal(amax, prev_amax))


def run_block(logits_for_step, seed, block, vocab, canvas_len, *, max_steps=MAX_STEPS,
              fixed_steps=None, tau=TAU, h_bound=H_BOUND, temperature=1.0, rule="confidence",
              entropy_bound=0.1, sticky=False):
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
    locked = None
    for t in range(1, n_steps + 1):
        logits = logits_for_step(t, canvas)
        conf, ent, amax = row_stats(logits, temperature)
        hbar = float(ent.mean())
        stop_now = would_stop(t, hbar, amax, prev, h_bound)
        nxt, locked = sample_update(conf, amax, seed, block, t, vocab, tau, entropy=ent, rule=rule,
                                    entropy_bound=entropy_bound, sticky=sticky,
                                    prev_canvas=canvas, prev_locked=locked)
        steps.append(dict(step=t, canvas_in=canvas, amax=amax, conf=conf, entropy=ent,
                          mean_entropy=hbar, locked=locked, canvas_out=nxt, stop=stop_now))
        if stop_now and first_stop is None:
            first_stop = t
        canvas = nxt
        prev = amax
        if stop_now and fixed_steps is None:
            stop_step = t
            break
    # a locked position commits its canvas token (its argmax unless a sticky lock kept an older
    # token), every other position its argmax
    last = steps[stop_step - 1]
    committed = np.where(last["locked"], last["canvas_out"], last["amax"])
    return dict(committed=committed, stop_step=stop_step, would_stop_step=first_stop, steps=steps,
                canvas=canvas)
