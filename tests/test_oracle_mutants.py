"""The oracle's pins are strong enough to catch plausible mistakes.

Each case plants one mistake in a copy of oracle/tide_oracle.c (on the CPU,
in a temporary directory), builds it, points the pin tests at it through
TIDE_ORACLE_LIB and checks that at least one pin fails.  Every mutation keeps
all memory accesses inside their buffers.  The mutants' pin runs are separate
processes, run a few at a time before the cases check their results.
"""
import concurrent.futures
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "tide_oracle.c")

MUTANTS = {
    "drops_last_rank": ("    for (int64_t k = 0; k < W; ++k) {\n        if (k == 0) {",
                        "    for (int64_t k = 0; k < W - 1; ++k) {\n        if (k == 0) {"),
    "subtracts_instead_of_adds": ("out[j] = out[j] + packed[j];", "out[j] = out[j] - packed[j];"),
    "rows_per_shard_off_by_one": ("S[i] = (d0[i] + W - 1) / W;", "S[i] = d0[i] / W + 1;"),
    "pack_uses_local_row": ("bf16_to_f32(g[i][row * inner[i] + t])", "bf16_to_f32(g[i][s * inner[i] + t])"),
    "scales_by_W_not_inverse": ("        float s = 1.0f / (float)W;\n        for (int64_t j = 0; j < n; ++j) out[j] = out[j] * s;",
                                "        float s = (float)W;\n        for (int64_t j = 0; j < n; ++j) out[j] = out[j] * s;"),
    "sum_starts_from_plus_zero": ("        if (k == 0) {\n            pack_f32(W, P, d0, inner, S, off, Ns, grads, out);\n        } else {",
                                  "        if (k == 0) for (int64_t j = 0; j < n; ++j) out[j] = 0.0f;\n        {"),
    "ag_pad_rows_not_zeroed": ("for (int64_t t = 0; t < inner[i]; ++t) dst[t] = 0;", ";"),
    "ag_source_stride_dropped": ("const uint16_t* src = ag + r * Ns + off[i] + s * inner[i];",
                                 "const uint16_t* src = ag + r * Ns + off[i] + s;"),
    "tree_pairs_mirrored": ("for (int64_t j = 0; j + 1 < n; j += 2) v[m++] = v[j] + v[j + 1];",
                            "for (int64_t j = 0; j + 1 < n; j += 2) v[m++] = v[j] + v[n - 1 - j];"),
    "tree_odd_one_dropped": ("if (n % 2 == 1) v[m++] = v[n - 1];", "if (n % 2 == 1) m += 0;"),
    "exact_magnitude_keeps_sign": ("mag += v < 0 ? -v : v;", "mag += v;"),
    "f32_pack_reads_bf16": ("dst[t] = row < d0[i] ? g[i][row * inner[i] + t] : 0.0f;",
                            "dst[t] = row < d0[i] ? bf16_to_f32(((const uint16_t*)g[i])[row * inner[i] + t]) : 0.0f;"),
    "f32_slots_drop_last_rank": ("for (int64_t k = 1; k < W; ++k) acc = acc + slots[k][j];",
                                 "for (int64_t k = 1; k < W - 1; ++k) acc = acc + slots[k][j];"),
    "f32_stage_writes_pad_rows": ("if (src_row >= d0[i]) continue;",
                                  "if (src_row >= d0[i]) { for (int64_t t = 0; t < inner[i]; ++t) "
                                  "slot[r * Ns + off[i] + s * inner[i] + t] = 0; continue; }"),
    "f32_stage_drops_row_stride": ("= g[i][src_row * inner[i] + t];", "= g[i][src_row + t * 0];"),
    "f32_scales_by_W_not_inverse": ("        float sc = 1.0f / (float)W;\n        for (int64_t j = 0; j < n; ++j) out[j] = out[j] * sc;",
                                    "        float sc = (float)W;\n        for (int64_t j = 0; j < n; ++j) out[j] = out[j] * sc;"),
    "ranks_added_in_reverse": ("pack_f32(W, P, d0, inner, S, off, Ns, grads + k * P, packed);",
                               "pack_f32(W, P, d0, inner, S, off, Ns, grads + (W - k) * P, packed);"),
}


def _run_mutant(name, root):
    """Build the mutant of `name` under `root` and run the pins against it; (returncode, output)."""
    old, new = MUTANTS[name]
    text = open(SRC).read()
    if text.count(old) != 1:
        return None, f"mutation anchor for {name} not unique"
    d = root / name
    d.mkdir()
    mutant_c = d / "mutant.c"
    mutant_c.write_text(text.replace(old, new))
    lib = d / "libmutant.so"
    subprocess.run(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared", "-o",
                    str(lib), str(mutant_c)], check=True)
    # one thread per pin process: the mutants run side by side
    env = dict(os.environ, TIDE_ORACLE_LIB=str(lib), OMP_NUM_THREADS="1", MKL_NUM_THREADS="1",
               OPENBLAS_NUM_THREADS="1")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        "-k", "not gloo", os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    return r.returncode, r.stdout


@pytest.fixture(scope="module")
def mutant_runs(tmp_path_factory):
    """Every mutant's pin run, several at a time (each is an independent process)."""
    root = tmp_path_factory.mktemp("mutants")
    names = sorted(MUTANTS)
    workers = max(1, min(len(names), (os.cpu_count() or 2) // 2))
    with concurrent.futures.ThreadPoolExecutor(max_workers=workers) as ex:
        return dict(zip(names, ex.map(lambda n: _run_mutant(n, root), names)))


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, mutant_runs):
    rc, out = mutant_runs[name]
    assert rc is not None, out
    assert rc != 0, f"no pin caught mutant {name}:\n{out[-2000:]}"
    assert "failed" in out or "Error" in out
