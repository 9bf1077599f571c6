"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a copy of the C oracle (a wrong head map, a dropped
ReLU, an off-by-one block count, the wrong tie order, a wrong mean divisor, a
transposed indexer query, a missing softmax scale, a dropped partial-block token,
ties rounded away from even, a draft query's tail starting at its own block or
ending at the selection's query) and runs the CPU pins against the copy: every planted
mistake must make them fail.  Only the copy under a temporary directory is changed.
"""

import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MUTATIONS = [
    ("head map", "const int32_t g = h / group;", "const int32_t g = h % group;"),
    ("ReLU dropped", "dot > 0.0 ? dot : 0.0", "dot"),
    ("block count", "const int64_t n_complete = (t + 1) / block_size;", "const int64_t n_complete = t / block_size;"),
    ("tie order", "return (a->block > b->block) - (a->block < b->block);",
     "return (a->block < b->block) - (a->block > b->block);"),
    ("mean divisor", "sum / (double)block_size", "sum / (double)(block_size + 1)"),
    ("transposed query", "qo_bf16_value(q_idx[h * idx_dim + d])", "qo_bf16_value(q_idx[d * n_idx_heads + h])"),
    ("softmax scale", "logit[j] = scale * dot;", "logit[j] = dot;"),
    ("partial block token", "for (int64_t p = n_complete * block_size; p <= t; ++p)",
     "for (int64_t p = n_complete * block_size; p < t; ++p)"),
    ("ties to even", "const double r = nearbyint(a / step);", "const double r = floor(a / step + 0.5);"),
    ("draft tail start", "const int64_t n_complete_sel = (t_sel + 1) / block_size;",
     "const int64_t n_complete_sel = (t + 1) / block_size;"),
    ("draft tail end", "for (int64_t p = n_complete_sel * block_size; p <= t; ++p)",
     "for (int64_t p = n_complete_sel * block_size; p <= t_sel; ++p)"),
]


def _pins_on_copy(tmp_path, good=None, bad=None):
    """Run the oracle pins on a copy of the oracle, optionally with good -> bad applied."""
    dst = tmp_path / "repo"
    dst.mkdir()
    for d in ("oracle", "qsa_synth"):
        shutil.copytree(os.path.join(ROOT, d), dst / d, ignore=shutil.ignore_patterns("*.so", "__pycache__"))
    (dst / "tests").mkdir()
    for f in ("conftest.py", "test_oracle_pins.py"):
        shutil.copy(os.path.join(ROOT, "tests", f), dst / "tests" / f)
    shutil.copytree(os.path.join(ROOT, "tests", "golden"), dst / "tests" / "golden")
    shutil.copy(os.path.join(ROOT, "pytest.ini"), dst / "pytest.ini")
    if good is not None:
        src = dst / "oracle" / "qsa_oracle.c"
        text = src.read_text()
        assert text.count(good) == 1, f"mutation site not found: {good}"
        src.write_text(text.replace(good, bad))
    return subprocess.run([sys.executable, "-m", "pytest", "tests/test_oracle_pins.py", "-q", "-x", "-p",
                           "no:cacheprovider"], cwd=dst, capture_output=True, text=True, timeout=600)


def test_pins_pass_on_an_unchanged_copy(tmp_path):
    r = _pins_on_copy(tmp_path)
    assert r.returncode == 0, r.stdout[-2000:]


@pytest.mark.parametrize("name,good,bad", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_pins_fail_on_planted_mistake(tmp_path, name, good, bad):
    r = _pins_on_copy(tmp_path, good, bad)
    assert r.returncode != 0, f"pins still pass with the mistake '{name}' planted:\n{r.stdout[-2000:]}"
