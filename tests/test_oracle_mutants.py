"""Plant plausible mistakes in a copy of the oracle and check that its pins
fail (CPU only).

Each case rewrites one line of a temporary copy of ``oracle/oracle.cpp`` or
``oracle/__init__.py`` (a flipped sign, a dropped term, a swapped operand, a
wrong rounding or layout rule), rebuilds it there, and runs the pin test that
must catch it.
The real oracle is never modified.
"""
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# name: (original line(s), planted mistake, pin test that must fail)
MUTANTS = {
    "m_sign": ("        m = m + t;", "        m = m - t;",
               "test_oracle_adam.py::test_golden_first_step"),
    "no_decay": ("        float pn = p[i] * c.decay;", "        float pn = p[i];",
                 "test_oracle_adam.py::test_golden_first_step"),
    "no_bias_corr2_step": ("    c.step_hat = (float)(l * sq2 / bc1);", "    c.step_hat = (float)(l / bc1);",
                           "test_oracle_adam.py::test_golden_first_step"),
    "no_bias_corr2_eps": ("    c.eps_hat = (float)(E * sq2);", "    c.eps_hat = (float)(E);",
                          "test_oracle_adam.py::test_first_step_closed_form"),
    "eps_inside_sqrt": ("        float d = r + c.eps_hat;", "        float d = std::sqrt(v + c.eps_hat);",
                        "test_oracle_adam.py::test_first_step_closed_form"),
    "m_dequant_255": ("    const float dqm = *sm / 127.0f;", "    const float dqm = *sm / 255.0f;",
                      "test_oracle_adam.py::test_uniform_magnitude_blocks_reduce_to_adamw"),
    "v_quant_127": ("    const float qv = amax_r > 0.0f ? 255.0f / amax_r : 0.0f;",
                    "    const float qv = amax_r > 0.0f ? 127.0f / amax_r : 0.0f;",
                    "test_oracle_adam.py::test_golden_first_step"),
    "truncate_codes": ("        float a = std::rint(mt[i] * qm);", "        float a = std::trunc(mt[i] * qm);",
                       "test_oracle_adam.py::test_first_step_codes_are_nearest_levels"),
    "v_not_squared": ("        float vo = so * so;", "        float vo = so;",
                      "test_oracle_adam.py::test_uniform_magnitude_blocks_reduce_to_adamw"),
    "beta_swap": ("        float m = c.b1 * mo;", "        float m = c.b2 * mo;",
                  "test_oracle_adam.py::test_uniform_magnitude_blocks_reduce_to_adamw"),
    "no_bias_corr1": ("    c.step_hat = (float)(l * sq2 / bc1);", "    c.step_hat = (float)(l * sq2);",
                      "test_oracle_adam.py::test_first_step_closed_form"),
    "coupled_decay": ("        float gi = bf16_to_f32(g[i]) * grad_scale;",
                      "        float gi = bf16_to_f32(g[i]) * grad_scale + 0.01f * p[i];",
                      "test_oracle_adam.py::test_first_step_closed_form"),
    "scale_not_absmax": ("    *sm = amax_m;", "    *sm = amax_m * 0.5f;",
                         "test_oracle_adam.py::test_first_step_codes_are_nearest_levels"),
    "bf16_truncates": ("    u += 0x7FFFu + ((u >> 16) & 1u);", "    u += 0;",
                       "test_oracle_adam.py::test_bf16_rounding_matches_torch"),
    "walk_skips_check": ("        if (j > 0 && start_allowed(R - j, n, b, s, m, A)) return R - j;",
                         "        if (j > 0) return R - j;",
                         "test_oracle_layout.py::test_greedy_places_iff_any_placement_exists"),
    "skip_rule_too_strong": ("        if (t.n > 2 * s && s % t.b != 0) return false;",
                             "        if (t.n > s && s % t.b != 0) return false;",
                             "test_oracle_layout.py::test_chosen_slice_is_smallest_feasible"),
    "sort_ascending": ("        if (x.b != y.b) return x.b > y.b;", "        if (x.b != y.b) return x.b < y.b;",
                       "test_oracle_layout.py::test_golden_tiny_layout"),
    "candidate_step_b": ("    const int64_t L = std::lcm(A, b);", "    const int64_t L = b;",
                         "test_oracle_layout.py::test_literal_scan_equals_walk"),
    "edge_counts_as_inside": ("    for (int64_t r = o / s + 1; r < m && r * s < o + n; ++r)",
                              "    for (int64_t r = o / s + 1; r < m && r * s <= o + n; ++r)",
                              "test_oracle_layout.py::test_literal_scan_equals_walk"),
    "tile_transposed": ("                for (int64_t q = 0; q < width[j]; ++q) at[r * width[j] + q] = base[j] + r * stride[j] + q;",
                        "                for (int64_t q = 0; q < width[j]; ++q) at[r * width[j] + q] = base[j] + q * stride[j] + r;",
                        "test_oracle_tiles.py::test_golden_tiles_first_step"),
}

# The same for the oracle's Python part (oracle/__init__.py).
PY_MUTANTS = {
    "rowwise_floor_rows": ("    q = (rows + m - 1) // m", "    q = rows // m",
                           "test_oracle_rowwise.py::test_golden_rowwise_layout"),
    "rowwise_inclusive_offsets": ("    off = np.concatenate([[0], np.cumsum(sizes)[:-1]]).astype(np.int64)",
                                  "    off = (np.cumsum(sizes) - sizes[0]).astype(np.int64)",
                                  "test_oracle_rowwise.py::test_golden_rowwise_layout"),
    "rowwise_rank_minor": ("            src = r * C + int(off[t])", "            src = int(off[t]) * m + r",
                           "test_oracle_rowwise.py::test_copy_out_inverts_copy_in"),
    "tiles_full_last_width": ("                width.append(min(W, C - c0))", "                width.append(W)",
                              "test_oracle_tiles.py::test_golden_tiles_first_step"),
    "tiles_rows_as_blocks": ("        W = C if int(bc[i]) <= 0 or int(bc[i]) >= C else int(bc[i])",
                             "        W = C",
                             "test_oracle_tiles.py::test_golden_tiles_first_step"),
    "ns_swap_bc": ("        B = b * A + c * (A @ A)", "        B = c * A + b * (A @ A)",
                   "test_oracle_muon.py::test_newton_schulz_is_the_spectral_map"),
    "ns_no_normalise": ("    X = X / (np.linalg.norm(X) + eps)", "    X = X",
                        "test_oracle_muon.py::test_newton_schulz_is_the_spectral_map"),
    "momentum_not_nesterov": ("    return t + b * mom if nesterov else mom.copy()", "    return mom.copy()",
                              "test_oracle_muon.py::test_momentum_of_a_constant_gradient"),
    "momentum_unscaled": ("    t = g * np.float32(grad_scale)", "    t = g",
                          "test_oracle_muon.py::test_momentum_of_a_constant_gradient"),
    "rank_not_rebased": ('        out["offsets"].append(a - lo)', '        out["offsets"].append(a - o)',
                         "test_oracle_rank_buckets.py::test_rank_buckets_step_like_the_whole_bucket"),
    "rank_first_block_floor": ("        first_block += tiles_per_row_block * (-(-first_row_in // K))",
                               "        first_block += tiles_per_row_block * (first_row_in // K)",
                               "test_oracle_rank_buckets.py::test_rank_buckets_step_like_the_whole_bucket"),
    "rank_first_block_rows_only": ("        first_block += tiles_per_row_block * (-(-first_row_in // K))",
                                   "        first_block += -(-first_row_in // K)",
                                   "test_oracle_rank_buckets.py::test_first_block_counts_the_blocks_before_the_slice"),
    "rank_tiles_dropped": ('        out["block_cols"].append(int(bc[i]))', '        out["block_cols"].append(0)',
                           "test_oracle_rank_buckets.py::test_rank_buckets_step_like_the_whole_bucket"),
    "rowwise_unscaled": ("            pack(g[r0 * int(cols[t]):r0 * int(cols[t]) + k], seg, scale)",
                         "            pack(g[r0 * int(cols[t]):r0 * int(cols[t]) + k], seg, 1.0)",
                         "test_oracle_rowwise.py::test_golden_rowwise_layout"),
}


ALL = {**{k: ("oracle.cpp",) + v for k, v in MUTANTS.items()},
       **{k: ("__init__.py",) + v for k, v in PY_MUTANTS.items()}}


@pytest.mark.parametrize("name", sorted(ALL))
def test_pin_catches_planted_mistake(name, tmp_path):
    fname, orig, bad, pin = ALL[name]
    src = open(os.path.join(ROOT, "oracle", fname)).read()
    assert src.count(orig) == 1, f"mutation site of {name} not found once"
    work = tmp_path / "repo"
    os.makedirs(work / "tests")
    # A mistake planted in the Python part keeps the built library (same
    # source); one in oracle.cpp is rebuilt from the edited copy.
    skip = ("__pycache__",) if fname != "oracle.cpp" else ("*.so", "__pycache__")
    shutil.copytree(os.path.join(ROOT, "oracle"), work / "oracle", ignore=shutil.ignore_patterns(*skip))
    shutil.copytree(os.path.join(ROOT, "synth"), work / "synth",
                    ignore=shutil.ignore_patterns("__pycache__"))
    for f in ("conftest.py", "test_oracle_adam.py", "test_oracle_layout.py", "test_oracle_rowwise.py",
              "test_oracle_tiles.py", "test_oracle_muon.py", "test_oracle_rank_buckets.py"):
        shutil.copy(os.path.join(ROOT, "tests", f), work / "tests" / f)
    shutil.copytree(os.path.join(ROOT, "tests", "golden"), work / "tests" / "golden")
    (work / "oracle" / fname).write_text(src.replace(orig, bad))
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        "tests/" + pin], cwd=work, capture_output=True, text=True, timeout=600)
    assert r.returncode == 1 and "failed" in r.stdout, (
        f"pin {pin} did not catch mutant {name}:\n{r.stdout[-2000:]}{r.stderr[-2000:]}")
