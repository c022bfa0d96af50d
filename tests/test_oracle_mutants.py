"""Mutation check of the oracle's pins: each case plants ONE plausible mistake in a
copy of the C oracle (a dropped term, a wrong sign, a transposed operand, an index
or shift slip, a missing document mask), builds it with the oracle's own flags,
and runs the pin suites against it.  At least one pin must fail for every mutant;
the unmutated copy, built the same way, must pass them all.

What each mutant breaks is the formula it names: "Dynamic Short Convolutions
Improve Transformers", gist.science technical summary, section "Dynamic Short
Convolutions" (Mechanism formula y = u + sum_j w[t,c,j] u[t-j,c]; the low-rank
and head-wise Parameterization; the residual Placement), its gradients, this
library's reading that a filter stays inside its packed document, the decode
step's rolling state, and the RoPE rotation (RoFormer, section 3.4.2) applied
after the QKV conv.
"""
import concurrent.futures
import os
import subprocess
import sys

import pytest

from oracle import oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PIN_SUITES = ["tests/test_oracle_pins.py", "tests/test_oracle_rope_pins.py", "tests/test_oracle_decode_pins.py"]

# (name, text in the C oracle, its replacement at every place it occurs)
MUTANTS = [
    ("fwd_drops_residual",
     "double acc = u[n * C + c];", "double acc = 0.0;"),
    ("fwd_taps_reversed",
     "if (n - j >= st[n]) acc += w[c * K + j] * u[(n - j) * C + c];",
     "if (n - j >= st[n]) acc += w[c * K + (K - 1 - j)] * u[(n - j) * C + c];"),
    ("fwd_ignores_document_bounds",
     "if (n - j >= st[n]) acc += w[c * K + j] * u[(n - j) * C + c];",
     "if (n - j >= 0) acc += w[c * K + j] * u[(n - j) * C + c];"),
    ("fwd_reads_future_token",
     "if (n - j >= st[n]) acc += w[c * K + j] * u[(n - j) * C + c];",
     "if (n - j >= st[n]) acc += w[c * K + j] * u[(n + j < N ? n + j : n) * C + c];"),
    ("lowrank_B_transposed",
     "BW[k * (C * K) + c * K + j]", "BW[k * (C * K) + j * C + c]"),
    ("lowrank_A_transposed_in_z",
     "acc += h[n * d + i] * A[i * r + k];", "acc += h[n * d + i] * A[k * d + i];"),
    ("headwise_W_transposed",
     "BW[i * (H * K) + q * K + j]", "BW[i * (H * K) + j * H + q]"),
    ("du_uses_own_filter_not_source_token",
     "filter_row(p, h, A, BW, n, z, w);\n                for (int64_t c = 0; c < C; ++c) du_out",
     "filter_row(p, h, A, BW, m, z, w);\n                for (int64_t c = 0; c < C; ++c) du_out"),
    ("du_drops_residual_gradient",
     "for (int64_t c = 0; c < C; ++c) du_out[i * C + c] = g[m * C + c];",
     "for (int64_t c = 0; c < C; ++c) du_out[i * C + c] = 0.0;"),
    ("du_ignores_document_bounds",
     "if (n >= N || m < st[n]) continue;", "if (n >= N) continue;"),
    ("dw_time_indices_swapped",
     "g[n * C + c] * u[(n - j) * C + c] : 0.0;", "g[(n - j) * C + c] * u[n * C + c] : 0.0;"),
    ("dz_wrong_sign",
     "for (int64_t j = 0; j < K; ++j) acc += dw[c * K + j] * BW[k * (C * K) + c * K + j];",
     "for (int64_t j = 0; j < K; ++j) acc -= dw[c * K + j] * BW[k * (C * K) + c * K + j];"),
    ("dh_A_transposed",
     "acc += dg[k] * A[a * p->rank + k];", "acc += dg[k] * A[k * d + a];"),
    ("dB_ignores_document_bounds",
     "if (n - j >= st[n]) acc += zall[n * r + k] * (g[n * C + c] * u[(n - j) * C + c]);",
     "if (n - j >= 0) acc += zall[n * r + k] * (g[n * C + c] * u[(n - j) * C + c]);"),
    ("dA_wrong_rank_column",
     "acc += h[n * d + a] * dgen[n * r + k];", "acc += h[n * d + a] * dgen[n * r + (r - 1 - k)];"),
    ("dwh_sums_neighbouring_head",
     "for (int64_t c = q * p->head_dim; c < (q + 1) * p->head_dim; ++c) acc += dw[c * K + j];",
     "for (int64_t c = q * p->head_dim; c < (q + 1) * p->head_dim; ++c) acc += dw[((c + p->head_dim) % C) * K + j];"),
    ("headwise_dh_wrong_column",
     "acc += dg[e] * BW[a * gdim(p) + e];", "acc += dg[e] * BW[a * gdim(p) + (gdim(p) - 1 - e)];"),
    ("dW_wrong_column",
     "acc += h[n * d + a] * dgen[n * G + col];", "acc += h[n * d + a] * dgen[n * G + (G - 1 - col)];"),
    ("dB_drops_shift",
     "acc += zall[n * r + k] * (g[n * C + c] * u[(n - j) * C + c]);",
     "acc += zall[n * r + k] * (g[n * C + c] * u[n * C + c]);"),
    ("z_drops_last_hidden_dim",
     "for (int64_t i = 0; i < d; ++i) acc += h[n * d + i] * A[i * r + k];",
     "for (int64_t i = 0; i < d - 1; ++i) acc += h[n * d + i] * A[i * r + k];"),
    ("fwd_drops_last_tap",
     "for (int64_t j = 0; j < K; ++j)\n                    if (n - j >= st[n]) acc += w",
     "for (int64_t j = 0; j < K - 1; ++j)\n                    if (n - j >= st[n]) acc += w"),
    ("du_drops_last_tap",
     "for (int64_t j = 0; j < K; ++j) {\n                const int64_t n = m + j;",
     "for (int64_t j = 0; j < K - 1; ++j) {\n                const int64_t n = m + j;"),
    ("dB_entry_drops_shift",
     "acc += zk * (g[n * C + c] * u[(n - j) * C + c]);", "acc += zk * (g[n * C + c] * u[n * C + c]);"),
    ("dA_entry_B_transposed",
     "BW[i1 * (C * K) + c * K + j]", "BW[i1 * (C * K) + j * C + c]"),
    ("dW_entry_drops_shift",
     "s += g[n * C + c] * u[(n - j) * C + c];", "s += g[n * C + c] * u[n * C + c];"),
    ("segment_start_one_token_early",
     "st[n] = p->cu_seqlens[s];", "st[n] = p->cu_seqlens[s] > 0 ? p->cu_seqlens[s] - 1 : 0;"),
    ("decode_state_read_oldest_first",
     "x[j] = state[(b * (K - 1) + (j - 1)) * C + c];", "x[j] = state[(b * (K - 1) + (K - 1 - j)) * C + c];"),
    ("decode_state_not_rolled",
     "state[(b * (K - 1) + j) * C + c] = x[j];", "state[(b * (K - 1) + j) * C + c] = x[j + 1];"),
    ("decode_drops_residual",
     "double acc = x[0];", "double acc = 0.0;"),
    ("rope_frequency_exponent_halved",
     "pow(base, -2.0 * (double)i / (double)hd)", "pow(base, -(double)i / (double)hd)"),
    ("rope_position_not_reset_per_document",
     "const double pos = (double)(n - st[n]);", "const double pos = (double)n;"),
    ("rope_pair_index_not_reset_per_head",
     "const int64_t i = (c % hd) / 2;", "const int64_t i = c / 2;"),
    ("rope_turns_the_wrong_way",
     "x[ri * C + c] = x0 * cs - x1 * sn;\n                x[ri * C + c + 1] = x0 * sn + x1 * cs;",
     "x[ri * C + c] = x0 * cs + x1 * sn;\n                x[ri * C + c + 1] = -x0 * sn + x1 * cs;"),
]


def _mutate(src: str, old: str, new: str) -> str:
    assert src.count(old) >= 1, f"mutation site not found: {old!r}"
    return src.replace(old, new)


def _run_pins(name: str, src_text: str, workdir: str):
    """Build one variant of the oracle and run the pin suites against it: (returncode, first failure)."""
    c_path = os.path.join(workdir, f"{name}.c")
    so_path = os.path.join(workdir, f"lib{name}.so")
    with open(c_path, "w") as f:
        f.write(src_text)
    O.compile_library(c_path, so_path)
    env = dict(os.environ, DYNCONV_ORACLE_LIB=so_path, OMP_NUM_THREADS="1")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider", *PIN_SUITES],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    failed = [ln for ln in r.stdout.splitlines() if ln.startswith("FAILED")]
    return r.returncode, (failed[0] if failed else r.stdout[-400:])


@pytest.fixture(scope="module")
def outcomes(tmp_path_factory):
    workdir = str(tmp_path_factory.mktemp("oracle_mutants"))
    with open(O._SRC) as f:
        src = f.read()
    jobs = {"unmutated": src}
    for name, old, new in MUTANTS:
        jobs[name] = _mutate(src, old, new)
        assert jobs[name] != src
    with concurrent.futures.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        futs = {name: ex.submit(_run_pins, name, text, workdir) for name, text in jobs.items()}
        return {name: fut.result() for name, fut in futs.items()}


def test_unmutated_copy_passes_every_pin(outcomes):
    rc, detail = outcomes["unmutated"]
    assert rc == 0, f"the pin suites fail on an unmutated copy of the oracle: {detail}"


@pytest.mark.parametrize("name", [m[0] for m in MUTANTS])
def test_every_planted_mistake_fails_a_pin(outcomes, name):
    rc, detail = outcomes[name]
    # pytest exit code 1: tests ran and at least one failed (2-5 would be a harness error)
    assert rc == 1, f"mutant {name} survived every pin (pytest exit {rc}): {detail}"
