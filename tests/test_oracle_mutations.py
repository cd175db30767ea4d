"""The oracle's pins catch plausible mistakes (CPU only).

Each case copies ``oracle/`` to a temporary directory, plants one mistake in
the copy (a dropped term, a wrong sign, an off-by-one index, swapped operands
or byte order, a wrong rounding mode) and runs the pin suites
``test_oracle_quant.py`` and ``test_oracle_attention.py`` against the copy in
a subprocess. The suites must fail for every mutant and pass for an
unmodified copy. The real ``oracle/`` is never modified.
"""
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PINS = ["tests/test_oracle_quant.py", "tests/test_oracle_attention.py"]

# (name, file, original text, mutated text)
MUTANTS = [
    ("round_floor", "quant.py", "np.clip(np.rint(t),", "np.clip(np.floor(t),"),
    ("scale_divisor", "quant.py", "s32 = np.divide(rng_, qmax, dtype=np.float32)",
     "s32 = np.divide(rng_, qmax + 1, dtype=np.float32)"),
    ("zero_point_from_max", "quant.py", "z16 = mn.astype(np.float16)", "z16 = mx.astype(np.float16)"),
    ("signed_zero_minimum", "quant.py", "mn = np.add(xg.min(axis=-1), np.float32(0), dtype=np.float32)",
     "mn = xg.min(axis=-1)"),
    ("dequant_sign", "quant.py", "return (u * s + z).reshape(n, d)", "return (u * s - z).reshape(n, d)"),
    ("pack_nibble_order", "quant.py", "<< np.uint8(bits * k)", "<< np.uint8(bits * (per - 1 - k))"),
    ("meta_pair_order", "quant.py", "pair = np.stack([s, z], axis=-1)", "pair = np.stack([z, s], axis=-1)"),
    ("segment_order", "layout.py", "o_cm = _align16(o_rc + p * self.code_row_r)",
     "o_cm = _align16(o_cc + p * self.code_row_r)"),
    ("slot_off_by_one", "layout.py", "slot = t % p\n", "slot = (t + 1) % p\n"),
    ("wrong_request_table", "layout.py", "page = int(table[b][t // p])", "page = int(table[0][t // p])"),
    ("drop_rope_term", "attention.py", "S = (qc @ C.T + qr @ R.T) * float(scale)", "S = (qc @ C.T) * float(scale)"),
    ("scale_one_term", "attention.py", "S = (qc @ C.T + qr @ R.T) * float(scale)",
     "S = qc @ C.T * float(scale) + qr @ R.T"),
    ("causal_off_by_one", "attention.py", "return max(0, int(seq_len) - s_q + 1 + i)",
     "return max(0, int(seq_len) - s_q + i)"),
    ("mask_inclusive", "attention.py", "valid = np.arange(T)[None, :] < L[:, None]",
     "valid = np.arange(T)[None, :] <= L[:, None]"),
    ("missing_normalisation", "attention.py", "o[live] = (p @ C) / l_", "o[live] = p @ C"),
    ("lse_without_log", "attention.py", "lse[live] = (m + np.log(l_))[:, 0]", "lse[live] = (m + l_)[:, 0]"),
    ("combine_weight_sign", "attention.py", "w = np.exp(lse_parts[:, live] - m[live][None, :])",
     "w = np.exp(m[live][None, :] - lse_parts[:, live])"),
    ("hybrid_visibility", "attention.py", "scale, Th + Lp)", "scale, Th + Lp + 1)"),
    ("hybrid_drops_history", "attention.py", "np.concatenate([Ch, Cp]), np.concatenate([Rh, Rp])",
     "np.concatenate([Ch[:0], Cp]), np.concatenate([Rh[:0], Rp])"),
    ("query_rows_order", "attention.py", "return qc_b.reshape(s_q * H, -1), qr_b.reshape(s_q * H, -1), L",
     "return qc_b.transpose(1, 0, 2).reshape(s_q * H, -1), qr_b.reshape(s_q * H, -1), L"),
]


def _run_pins(tmp_path, mutant=None):
    dst = tmp_path / "oracle"
    shutil.copytree(os.path.join(ROOT, "oracle"), dst, ignore=shutil.ignore_patterns("__pycache__", "*.so", "*.o"))
    if mutant is not None:
        _, fname, old, new = mutant
        path = dst / fname
        src = path.read_text()
        assert src.count(old) == 1, f"mutation site not unique in {fname}: {old!r}"
        path.write_text(src.replace(old, new))
    driver = (
        "import sys\n"
        f"sys.path.insert(0, {str(tmp_path)!r})\n"
        "import oracle\n"
        f"assert oracle.__file__.startswith({str(tmp_path)!r}), oracle.__file__\n"
        "import pytest\n"
        f"sys.exit(pytest.main({PINS!r} + ['-x', '-q', '-p', 'no:cacheprovider', '-m', 'not gpu']))\n"
    )
    env = dict(os.environ, PYTHONDONTWRITEBYTECODE="1")
    r = subprocess.run([sys.executable, "-c", driver], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=600)
    return r.returncode, r.stdout[-2000:] + r.stderr[-2000:]


def test_unmodified_copy_passes(tmp_path):
    rc, log = _run_pins(tmp_path)
    assert rc == 0, log


@pytest.mark.parametrize("mutant", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, mutant):
    rc, log = _run_pins(tmp_path, mutant)
    assert rc == 1, f"pins did not catch mutant {mutant[0]} (exit {rc}):\n{log}"
