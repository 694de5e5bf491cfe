"""Plant plausible mistakes in a private copy of the oracle (on the CPU) and
check that the pins in ``test_oracle_pins`` catch every one of them."""

import inspect
import types

import pytest

import oracle.ress_oracle as ress_oracle
import tests.test_oracle_pins as pins

MUTATIONS = {
    "block sum instead of block mean":
        ("return np.ascontiguousarray((sums / block).transpose(1, 0, 2))",
         "return np.ascontiguousarray((sums).transpose(1, 0, 2))"),
    "temperature sqrt(8) regardless of d":
        ("return np.matmul(qbar, kbar.transpose(0, 2, 1)) / math.sqrt(d)",
         "return np.matmul(qbar, kbar.transpose(0, 2, 1)) / math.sqrt(8)"),
    "contrast against the next block":
        ("c[:, 1:] = np.sqrt((diff * diff).sum(axis=-1))",
         "c[:, :-1] = np.sqrt((diff * diff).sum(axis=-1))"),
    "ties to the higher index":
        ('order = np.argsort(-score, axis=-1, kind="stable")[..., :budget]',
         'order = (score.shape[-1] - 1 - np.argsort(-score[..., ::-1], axis=-1, kind="stable"))[..., :budget]'),
    "contrast as a factor":
        ("score = probs + lam * contrast[:, None, :]",
         "score = probs * (1 + lam * contrast[:, None, :])"),
    "lse without the row max":
        ("lse = m[:, 0] + np.log(l[:, 0])", "lse = np.log(l[:, 0])"),
    "drift with a shifted normaliser":
        ("w = np.exp(s - lse_blk[:, None]).reshape(q_blk.shape[0], nd, block)",
         "w = np.exp(s - lse_blk[:, None] - 0.01).reshape(q_blk.shape[0], nd, block)"),
    "drift as max-abs instead of Frobenius":
        ("drift = np.sqrt((contrib * contrib).sum(axis=(1, 2)))",
         "drift = np.abs(contrib).max(axis=(1, 2))"),
    "set drift as the sum of magnitudes":
        ("return drift, float(np.sqrt((total * total).sum()))",
         "return drift, float(drift.sum())"),
    "CDF threshold exceeded instead of reached":
        ("reached = cum >= tau", "reached = cum > tau"),
    "CDF count off by one":
        ("first = np.argmax(reached, axis=-1) + 1", "first = np.argmax(reached, axis=-1)"),
    "CDF over ascending probabilities":
        ('order = np.argsort(-p, axis=-1, kind="stable")', 'order = np.argsort(p, axis=-1, kind="stable")'),
    "padding pooled into the block means":
        ("w = valid.reshape(nb, block).astype(np.float64)", "w = np.ones((nb, block))"),
    "padding keys enter the softmax":
        ("keys = valid if special[t] else (valid & kept_tok)",
         "keys = np.ones(n, dtype=bool) if special[t] else kept_tok"),
    "special queries follow the sparse mask":
        ("keys = valid if special[t] else (valid & kept_tok)", "keys = valid & kept_tok"),
    "special-only key blocks not forced":
        ("rank[:, :, forced] = np.inf", "rank[:, :, forced] = rank[:, :, forced]"),
    "special queries counted in the drift":
        ("live = valid[rows] & ~special[rows]", "live = valid[rows]"),
    "padding keys in the drift":
        ("toks = toks[valid[toks]]", "toks = toks"),
    "empty key blocks ranked like the others":
        ("rank[:, :, empty] = -np.inf", "rank[:, :, empty] = rank[:, :, empty]"),
    "restoration accepts swaps that raise J":
        ("        if not jnew < jcur:\n            break", "        if jnew > jcur + 1e30:\n            break"),
    "pooled contribution without the probability":
        ("return sc[\"probs\"][..., None] * vbar[:, None, :, :]",
         "return 0.0 * sc[\"probs\"][..., None] + vbar[:, None, :, :]"),
    "drop-set drift as the sum of magnitudes":
        ("return float(np.linalg.norm(c[drop].sum(axis=0)))",
         "return float(np.linalg.norm(c[drop], axis=1).sum())"),
    "initial set of lowest drift score":
        ("order = np.argsort(-score, kind=\"stable\")", "order = np.argsort(score, kind=\"stable\")"),
    "restoration candidates by the wrong sign":
        ("out = sorted(drop, key=lambda b: (-gain[b], b))[:cand]",
         "out = sorted(drop, key=lambda b: (gain[b], b))[:cand]"),
    "a causal mask over the kept tokens":
        ("s = (q_blk @ keys.T) / math.sqrt(d)\n    m = s.max",
         "s = (q_blk @ keys.T) / math.sqrt(d)\n    s = s + np.triu(np.full(s.shape, -np.inf), 1)\n    m = s.max"),
    "VASC contrast as the L2 norm instead of the RMS":
        ("rho[:, p] = np.sqrt((diff * diff).sum(axis=-1) / d)",
         "rho[:, p] = np.sqrt((diff * diff).sum(axis=-1))"),
    "VASC sliding pairs instead of fixed ones":
        ("diff = vbar[:, 2 * p, :] - vbar[:, 2 * p + 1, :]",
         "diff = vbar[:, p, :] - vbar[:, p + 1, :]"),
    "VASC singleton averaged over two children":
        ("        size[-1] = 1", "        size[-1] = 2"),
    "VASC demand not clipped at one":
        ("a[h, i] = np.minimum(1.0, c * d / total)", "a[h, i] = c * d / total"),
    "VASC demand rescaled to one instead of the capacity":
        ("a[h, i] = np.minimum(1.0, c * d / total)", "a[h, i] = np.minimum(1.0, d / total)"),
    "VASC contrast added to the relevance":
        ("d = p[h, i] * factor[h]", "d = p[h, i] + factor[h]"),
    "VASC memory normalised over all heads":
        ("top = m[h].max() if m.shape[1] else 0.0", "top = m.max() if m.shape[1] else 0.0"),
    "VASC memory ignored by the ranking":
        ("score = demand + mhat[:, None, pair_of]", "score = demand + 0.0 * mhat[:, None, pair_of]"),
    "VASC deficit not clipped at zero":
        ("mem_out = np.maximum(0.0, mem_in + dmean - smean)", "mem_out = mem_in + dmean - smean"),
    "VASC memory adds service and subtracts demand":
        ("mem_out = np.maximum(0.0, mem_in + dmean - smean)",
         "mem_out = np.maximum(0.0, mem_in - dmean + smean)"),
}


def _mutant(old, new):
    src = inspect.getsource(ress_oracle)
    assert old in src, old
    mod = types.ModuleType("oracle_mutant")
    exec(compile(src.replace(old, new), "oracle_mutant", "exec"), mod.__dict__)
    return mod


def _pin_tests():
    return [getattr(pins, n) for n in dir(pins) if n.startswith("test_")]


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(name, monkeypatch):
    mutant = _mutant(*MUTATIONS[name])
    monkeypatch.setattr(pins, "oracle", mutant)
    caught = []
    for fn in _pin_tests():
        try:
            fn()
        except Exception:   # noqa: BLE001 - any failure counts as caught
            caught.append(fn.__name__)
    assert caught, f"no pin caught: {name}"


def test_unmutated_oracle_passes_every_pin():
    for fn in _pin_tests():
        fn()
