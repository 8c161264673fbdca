"""The pins catch planted mistakes (CPU). Each case plants one plausible
mistake in a scratch copy of the oracle, such as a dropped term, a wrong sign,
a wrong index, a transposed gather or a swapped operand. It then runs the
oracle's pins against that copy, which must fail. Only the copy is changed;
the oracle in the repository is never touched."""
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# (what the mistake is, text in oracle/attention.py, its replacement)
MUTATIONS = [
    ("sink left out of the denominator", "Z += math.exp(sinks[r] - m)", "Z += 0.0"),
    ("sink sign flipped", "Z += math.exp(sinks[r] - m)", "Z += math.exp(-sinks[r] - m)"),
    ("causal not bottom-right", "hi = min(hi, i + delta)\n", "hi = min(hi, i)\n"),
    ("left window bound off by one", "lo = max(lo, i + delta - window_left)",
     "lo = max(lo, i + delta - window_left + 1)"),
    ("GQA heads interleaved", "return h // (num_heads_q // num_heads_kv)",
     "return h % num_heads_kv"),
    ("scale dropped", "s = scale * (q @ k.T)", "s = (q @ k.T)"),
    ("LSE includes the sink", "lse[r] = M + math.log(np.exp(sj - M).sum())",
     "lse[r] = m + math.log(Z)"),
    ("e4m3 exponent bias wrong", "normal = sign * np.ldexp(1.0 + m / 8.0, (e - 7)",
     "normal = sign * np.ldexp(1.0 + m / 8.0, (e - 8)"),
    ("page row taken from the page index", "return cache[blocks, idx % page]",
     "return cache[blocks, idx // page]"),
    ("combine weights inverted", "np.exp(Ls - Msafe[None])", "np.exp(Msafe[None] - Ls)"),
    ("MLA V taken from the row's end", "kv[..., :head_dim_v]", "kv[..., -head_dim_v:]"),
    ("q descale divides", "qs = qs * float(q_descale[b][g])",
     "qs = qs / float(q_descale[b][g])"),
    ("appended keys put first", "ks = np.concatenate([ks, np.asarray(k_new[b], np.float64)])",
     "ks = np.concatenate([np.asarray(k_new[b], np.float64), ks])"),
    ("sparse block index not scaled", "idx[:, None] * block_size + np.arange(block_size)",
     "idx[:, None] + np.arange(block_size)"),
    ("sparse causal not bottom-right", "idx = idx[idx <= i + L - Sq]", "idx = idx[idx <= i]"),
    ("additive mask dropped", "s = s + np.asarray(bias, dtype=np.float64)", "s = s"),
    ("MLA K and V descales swapped", "None, rows, q_descale, k_descale, v_descale)",
     "None, rows, q_descale, v_descale, k_descale)"),
    ("sparse MLA V scaled by the K descale", "qs, ks, vs = qs * dq, ks * dk, vs * dv",
     "qs, ks, vs = qs * dq, ks * dk, vs * dk"),
]


@pytest.mark.parametrize("what,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_pins_catch_planted_mistake(tmp_path, what, old, new):
    src = os.path.join(ROOT, "oracle", "attention.py")
    text = open(src).read()
    assert text.count(old) == 1, f"mutation anchor not found once: {old!r}"
    shutil.copytree(os.path.join(ROOT, "oracle"), tmp_path / "oracle")
    (tmp_path / "oracle" / "attention.py").write_text(text.replace(old, new))
    shutil.copytree(os.path.join(ROOT, "tests"), tmp_path / "tests",
                    ignore=shutil.ignore_patterns("__pycache__", "test_oracle_mutations.py"))
    shutil.copy(os.path.join(ROOT, "pytest.ini"), tmp_path / "pytest.ini")
    env = dict(os.environ, PYTHONPATH=str(tmp_path), PYTHONDONTWRITEBYTECODE="1")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        "tests/test_oracle_pins.py", "tests/test_oracle_properties.py"],
                       cwd=tmp_path, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"the pins did not catch: {what}\n{r.stdout[-2000:]}"
    assert "failed" in r.stdout, r.stdout[-2000:]
