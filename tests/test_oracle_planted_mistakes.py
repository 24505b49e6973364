"""The oracle's pins catch plausible mistakes.

Each case below plants one mistake in a copy of the oracle's source (a
swapped index, a dropped term, an off-by-one bound, a wrong weighting), loads
that copy as a separate module, and runs the pins of one test module against
it in-process (the pin module's `oracle` name is pointed at the copy for the
duration).  At least one pin must then fail with an assertion.  The oracle
itself is never modified; every case also checks that the text it replaces
occurs exactly once, so an edit of the oracle that moves the text makes the
case fail loudly instead of passing vacuously.
"""
import importlib
import inspect
import itertools
import os
import types

import pytest

from conftest import ROOT

ORACLE_SRC = os.path.join(ROOT, "oracle", "ulysses_oracle.py")

ATT, RLY, KV, RING, LOSS = ("test_oracle_attention", "test_oracle_relayout", "test_oracle_kv_replication",
                            "test_oracle_ring", "test_oracle_loss")

# (what is wrong, text in the oracle, replacement, pin module expected to notice)
PLANTED = [
    ("seq->head: heads dealt round-robin", "src_head = np.broadcast_to(r * h + j, (P, n, h))",
     "src_head = np.broadcast_to(j * P + r, (P, n, h))", RLY),
    ("seq->head: ranks' chunks in reverse order", "src_rank = np.broadcast_to(t // m, (P, n, h))",
     "src_rank = np.broadcast_to((P - 1) - t // m, (P, n, h))", RLY),
    ("head->seq: token blocks reversed", "src_tok = np.broadcast_to(s * m + u, (P, m, H))",
     "src_tok = np.broadcast_to((P - 1 - s) * m + u, (P, m, H))", RLY),
    ("head->seq window: tokens interleaved", "np.broadcast_to(s * m + u, shape)",
     "np.broadcast_to(u * P + s, shape)", RLY),
    ("seq->head window: heads dealt round-robin", "np.broadcast_to(r * h + j, shape)]",
     "np.broadcast_to(r + j * P, shape)]", RLY),
    ("sharding: strided instead of contiguous chunks",
     "return np.stack([x[:, i * m:(i + 1) * m] for i in range(P)])",
     "return np.stack([x[:, i::P] for i in range(P)])", ATT),
    ("shape rule: H_q % H_kv not enforced", "    if h_q % h_kv:\n        raise", "    if False:\n        raise", RLY),
    ("sp sizes: H itself left out", "return [P for P in range(1, H + 1) if H % P == 0]",
     "return [P for P in range(1, H) if H % P == 0]", RLY),
    ("kv replication: head r mod H_kv", "return (r * H_kv) // P", "return r % H_kv", KV),
    ("kv reduce: last copy overwrites the sum", "out[s_, :, :, g] += x_head[r, :, s_ * m:(s_ + 1) * m, 0]",
     "out[s_, :, :, g] = x_head[r, :, s_ * m:(s_ + 1) * m, 0]", KV),
    ("layer backward: replicated dK halved",
     "kv_head_to_seq_reduce(dK, P, H_kv), kv_head_to_seq_reduce(dV, P, H_kv)",
     "kv_head_to_seq_reduce(dK, P, H_kv) * (0.5 if H_kv < P else 1.0), kv_head_to_seq_reduce(dV, P, H_kv)", KV),
    ("segments: token 0 not a sample start", "    flag[..., 0] = True\n", "", ATT),
    ("segments: start off by one", "idx = np.where(flag, np.arange(n), 0)",
     "idx = np.where(flag, np.arange(n) + 1, 0)", ATT),
    ("segments: end includes the next start",
     "shifted = np.concatenate([nxt[..., 1:], np.full(nxt.shape[:-1] + (1,), n)], axis=-1)", "shifted = nxt", ATT),
    ("mask: strictly causal (no diagonal)", "(i[None, :] <= i[:, None])", "(i[None, :] < i[:, None])", ATT),
    ("scale 1/d instead of 1/sqrt(d)", "return 1.0 / math.sqrt(d)", "return 1.0 / d", ATT),
    ("brute LSE without the max", "return Pm @ v, m[:, 0] + np.log(l[:, 0])", "return Pm @ v, np.log(l[:, 0])", ATT),
    ("brute backward: Jacobian summed over the wrong axis",
     "dS = Pm * (dP - (Pm * dP).sum(axis=1, keepdims=True))",
     "dS = Pm * (dP - (Pm * dP).sum(axis=0, keepdims=True))", ATT),
    ("brute backward: dK without the scale", "return scale * (dS @ k), scale * (dS.T @ q), dV",
     "return scale * (dS @ k), (dS.T @ q), dV", ATT),
    ("blocked: every row masked from the block's first sample start",
     "ok = (jj >= seg_start[i0:i1, None]) & (jj <= ii)", "ok = (jj >= seg_start[i0]) & (jj <= ii)", ATT),
    ("blocked: log1p for log in the LSE", "lse[i0 - row_lo:i1 - row_lo] = m + np.log(l)",
     "lse[i0 - row_lo:i1 - row_lo] = m + np.log1p(l)", ATT),
    ("blocked backward: D dropped", "D = (dO[i0:i1] * O).sum(axis=1)", "D = 0 * (dO[i0:i1] * O).sum(axis=1)", ATT),
    ("blocked backward: dK without the scale", "dK[lo:i1] += scale * (dS.T @ q[i0:i1])",
     "dK[lo:i1] += (dS.T @ q[i0:i1])", ATT),
    ("blocked backward: dV off by 0.1%", "dV[lo:i1] += Pm.T @ dO[i0:i1]",
     "dV[lo:i1] += Pm.T @ dO[i0:i1] * (1 + 1e-3)", ATT),
    ("row-sampled forward: output off by 1e-4", "acc += E @ v[c0:c1]", "acc += E @ v[c0:c1] * 1.0001", ATT),
    ("row-sampled backward: D dropped", "dQ += scale * ((Pm * (dP - D[:, None])) @ k[c0:c1])",
     "dQ += scale * ((Pm * dP) @ k[c0:c1])", ATT),
    ("GQA: query head h reads kv head h mod H_kv",
     "            g = h // G\n            if brute:\n                o, l",
     "            g = h % h_kv\n            if brute:\n                o, l", ATT),
    ("GQA backward: group gradients overwritten, not summed", "            dK[bb, :, g] += bk",
     "            dK[bb, :, g] = bk", ATT),
    ("per-rank forward: kv head j mod h_kv",
     "o, l = attention_fwd_head(q_head[r, bb, :, j], k_head[r, bb, :, j // G],",
     "o, l = attention_fwd_head(q_head[r, bb, :, j], k_head[r, bb, :, j % hkv],", ATT),
    ("per-rank backward: dV overwritten, not summed",
     "                dV[r, bb, :, g] += c\n    return dQ, dK, dV\n\n\ndef ulysses_layer_fwd",
     "                dV[r, bb, :, g] = c\n    return dQ, dK, dV\n\n\ndef ulysses_layer_fwd", ATT),
    ("single-rank mode computes the mirrored rank",
     "return range(P) if rank is None or rank < 0 else [rank]",
     "return range(P) if rank is None or rank < 0 else [P - 1 - rank]", ATT),
    ("key block: LSE without the max", "Lb[has] = m[has] + np.log(l[has])", "Lb[has] = np.log(l[has])", RING),
    ("key block: k_hi inclusive",
     "        hi = np.minimum(rows + 1, k_hi)\n        j0, j1 = int(lo.min()), int(hi.max())\n"
     "        if j1 <= j0:\n            continue\n        cols = np.arange(j0, j1)\n"
     "        vis = (cols[None, :] >= lo[:, None]) & (cols[None, :] < hi[:, None])\n        has",
     "        hi = np.minimum(rows + 1, k_hi + 1)\n        j0, j1 = int(lo.min()), int(hi.max())\n"
     "        if j1 <= j0:\n            continue\n        cols = np.arange(j0, j1)\n"
     "        vis = (cols[None, :] >= lo[:, None]) & (cols[None, :] < hi[:, None])\n        has", RING),
    ("key-block backward: D dropped", "D = np.sum(dO * O, axis=1)", "D = 0 * np.sum(dO * O, axis=1)", RING),
    ("key-block backward: dV scaled", "dV[j0:j1] += Pm.T @ dO[i0:i1]", "dV[j0:j1] += scale * (Pm.T @ dO[i0:i1])",
     RING),
    ("merge: exp(LSE) formed without the max shift",
     "total += np.where(np.isfinite(lse_parts[bk]), np.exp(lse_parts[bk] - msafe), 0.0)",
     "total += np.where(np.isfinite(lse_parts[bk]), np.exp(lse_parts[bk]) * np.exp(-msafe), 0.0)", RING),
    ("merge: weights normalised by the max, not the LSE",
     "w = np.where(fin & np.isfinite(lse_parts[bk]), np.exp(lse_parts[bk] - np.where(fin, lse, 0.0)), 0.0)",
     "w = np.where(fin & np.isfinite(lse_parts[bk]), np.exp(lse_parts[bk] - np.where(fin, m, 0.0)), 0.0)", RING),
    ("loss: token id 0 not counted", "counts[r] = int(np.count_nonzero(lab[r] != ignore_index))",
     "counts[r] = int(np.count_nonzero(lab[r] > 0))", LOSS),
    ("loss: every negative label excluded", "counts[r] = int(np.count_nonzero(lab[r] != ignore_index))",
     "counts[r] = int(np.count_nonzero(lab[r] >= 0))", LOSS),
    ("loss: no max(G, 1)", "denom = float(max(int(good.sum()), 1))",
     "denom = float(int(good.sum())) or float('nan')", LOSS),
    ("loss: ranks without valid labels not skipped",
     "        if good[r] > 0:\n            total += losses[r] * float(good[r])",
     "        if True:\n            total += losses[r] * float(good[r])", LOSS),
    ("loss: uniform gradient", "grad[r] = float(good[r]) / denom", "grad[r] = 1.0 / P", LOSS),
    ("loss: plain mean of rank losses", "    loss = total / denom\n", "    loss = float(np.mean(losses))\n", LOSS),
]


def _planted_module(old=None, new=None) -> types.ModuleType:
    """A fresh copy of the oracle module with `old` replaced by `new` (no
    replacement when old is None)."""
    src = open(ORACLE_SRC).read()
    if old is not None:
        assert src.count(old) == 1, f"planted text occurs {src.count(old)} times; update this case"
        src = src.replace(old, new)
    mod = types.ModuleType("oracle_with_planted_mistake")
    exec(compile(src, "<oracle with a planted mistake>", "exec"), mod.__dict__)
    return mod


def _param_sets(fn):
    """Keyword sets of a pin's stacked @pytest.mark.parametrize decorators."""
    axes = []
    for mark in getattr(fn, "pytestmark", []):
        if mark.name != "parametrize":
            continue
        names, values = mark.args[0], mark.args[1]
        names = [s.strip() for s in names.split(",")] if isinstance(names, str) else list(names)
        axes.append([dict(zip(names, (v,) if len(names) == 1 else tuple(v))) for v in values])
    for combo in itertools.product(*axes):
        kw = {}
        for part in combo:
            kw.update(part)
        yield kw


def _first_failing_pin(module_name: str, planted: types.ModuleType):
    pins = importlib.import_module(module_name)
    saved = pins.oracle
    pins.oracle = planted
    try:
        for name, fn in inspect.getmembers(pins, inspect.isfunction):
            if not name.startswith("test_") or fn.__module__ != pins.__name__:
                continue
            for kw in _param_sets(fn):
                if set(inspect.signature(fn).parameters) - set(kw):
                    break                                   # needs fixtures: not a plain pin
                try:
                    fn(**kw)
                except (AssertionError, pytest.fail.Exception):     # an assert, or pytest.raises unmet
                    return name
                except (ValueError, IndexError, FloatingPointError, ZeroDivisionError):
                    continue                                # a crash is not what this checks
        return None
    finally:
        pins.oracle = saved


@pytest.mark.filterwarnings("ignore::RuntimeWarning")
@pytest.mark.parametrize("what,old,new,module", PLANTED, ids=[p[0] for p in PLANTED])
def test_a_planted_mistake_fails_a_pin(what, old, new, module):
    planted = _planted_module(old, new)
    assert _first_failing_pin(module, planted) is not None, f"no pin in {module} notices: {what}"


@pytest.mark.parametrize("module", [ATT, RLY, KV, RING, LOSS])
def test_the_unaltered_copy_passes_every_pin(module):
    """Control: the same machinery with nothing planted finds no failure."""
    assert _first_failing_pin(module, _planted_module()) is None
