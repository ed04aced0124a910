"""The oracle's pins catch plausible mistakes.

Each case copies the oracle's C source to a temporary directory, plants one
mistake (a dropped term, a wrong sign or index, a transposed operand, a wrong
tie-break ...), builds it on the CPU and runs the pin suite against the mutant.
At least one pin must fail for every mutant.  The real oracle is not touched.
"""
import os
import tempfile

import pytest

import oracle as oracle_pkg
import test_oracle_pins as pins

MUTANTS = {
    "score drops the min statistic": ("for (int64_t s = 0; s < 3; ++s)",
                                      "for (int64_t s = 0; s < 2; ++s)"),
    "projection uses W transposed": ("Wh[ci * d + co]", "Wh[co * d + ci]"),
    "score pairs q with itself": ("acc += q[s * d + c] * kk[s * d + c];",
                                  "acc += q[s * d + c] * q[s * d + c];"),
    "tie goes to the higher index": ("if (a->j < b->j) return -1;\n    if (a->j > b->j) return 1;",
                                     "if (a->j < b->j) return 1;\n    if (a->j > b->j) return -1;"),
    "Top-k keeps the lowest scores": ("if (a->v > b->v) return -1;\n    if (a->v < b->v) return 1;",
                                      "if (a->v > b->v) return 1;\n    if (a->v < b->v) return -1;"),
    "softmax ignores the scale": ("double z = scale * dot;", "double z = dot;"),
    "softmax is not normalised": ("double p = logit[e] / denom;", "double p = logit[e];"),
    "lse drops the running max": ("lse_out[u * Bt + r] = mx + log(denom);",
                                  "lse_out[u * Bt + r] = log(denom);"),
    "tokens in column-major order": ("return (t * Hs + y) * Ws + x;",
                                     "return (t * Ws + x) * Hs + y;"),
    "tile grid rows and columns swapped": ("int64_t b = (j / nw) % nh;\n    int64_t c = j % nw;",
                                           "int64_t b = j % nh;\n    int64_t c = (j / nh) % nw;"),
    "avg divides by Bt + 1": ("out[0 * d + c] = sum / (double)Bt;",
                              "out[0 * d + c] = sum / (double)(Bt + 1);"),
    "max and min swapped": ("out[1 * d + c] = mx;\n            out[2 * d + c] = mn;",
                            "out[1 * d + c] = mn;\n            out[2 * d + c] = mx;"),
    "teacher average-pools": ("if (p > trow[j]) trow[j] = p;", "trow[j] += p / (double)Bt;"),
    "recall counts predicted tiles twice": ("hits += found;", "hits += found + (a == 0);"),
    "distillation gradient has the wrong sign": (
        "G[row * nT + j] = (exp(logp) - tg) / (tau * (double)R);",
        "G[row * nT + j] = (tg - exp(logp)) / (tau * (double)R);"),
    "distillation gradient drops the temperature": (
        "G[row * nT + j] = (exp(logp) - tg) / (tau * (double)R);",
        "G[row * nT + j] = (exp(logp) - tg) / ((double)R);"),
    "distillation uses the key stats for dWq": (
        "dWq[(h * d + ci) * d + co] += sq[ci] * dq[s3 * d + co];",
        "dWq[(h * d + ci) * d + co] += sk[ci] * dq[s3 * d + co];"),
    "distillation target not normalised": ("double tg = t[j] / tsum;", "double tg = t[j];"),
    # reversed divergence KL(estimator || target), with its own consistent
    # gradient: the chain-rule and finite-difference pins cannot see it
    "distillation KL reversed (loss and gradient)": (
        """            if (tg > 0.0) kl += tg * (log(tg) - logp);
            G[row * nT + j] = (exp(logp) - tg) / (tau * (double)R);
        }""",
        """            kl += exp(logp) * (logp - log(tg));
        }
        for (int64_t j = 0; j < nT; ++j) {
            double logp = s[j] / tau - lse;
            double tg = t[j] / tsum;
            G[row * nT + j] = exp(logp) * (logp - log(tg) - kl) / (tau * (double)R);
        }"""),
    # the row terms summed instead of averaged, gradient scaled to match
    "distillation sums the rows (loss and gradient)": (
        """            G[row * nT + j] = (exp(logp) - tg) / (tau * (double)R);
        }
        total += kl;""",
        """            G[row * nT + j] = (exp(logp) - tg) / tau;
        }
        total += kl * (double)R;"""),
    "e4m3 ties go to the lower code": ("code = (lo & 1) ? lo + 1 : lo;", "code = lo;"),
    "e4m3 exponent bias 8": ("v = ldexp(1.0 + (double)m / 8.0, e - 7);",
                             "v = ldexp(1.0 + (double)m / 8.0, e - 8);"),
    "e4m3 scale from the mean magnitude": ("if (a > amax) amax = a;", "amax += a / (float)n;"),
}


def pin_suite(o):
    """Every pin, run against oracle object ``o``; stops at the first failure."""
    yield lambda: pins.test_hand_example(o)
    for grid, shape in (((20, 48, 80), (4, 4, 8)), ((2, 6, 6), (2, 3, 2))):
        yield lambda g=grid, s=shape: pins.test_tiles_partition_grid_into_boxes(o, g, s)
    for case in pins.SMALL_CASES:
        yield lambda c=case: pins.test_tripool_brute_force(o, *c)
        yield lambda c=case: pins.test_score_brute_force(o, *c)
        yield lambda c=case: pins.test_attention_brute_force_token_mask(o, *c)
    yield lambda: pins.test_tripool_invariants(o)
    yield lambda: pins.test_tripool_constant_tiles(o)
    yield lambda: pins.test_projection_identity_and_linearity(o)
    yield lambda: pins.test_score_reduces_to_average_pooling(o)
    yield lambda: pins.test_topk_matches_stable_sort_and_counts(o)
    yield lambda: pins.test_topk_tie_goes_to_lower_index(o)
    yield lambda: pins.test_attention_all_tiles_is_dense_softmax(o)
    yield lambda: pins.test_attention_1d_tiles_is_block_sparse(o)
    yield lambda: pins.test_attention_renormalisation(o)
    yield lambda: pins.test_teacher_is_tile_max_of_dense_probs(o, *pins.SMALL_CASES[0])
    yield lambda: pins.test_tile_recall_hand_cases(o)
    yield lambda: pins.test_tile_recall_brute_force(o)
    yield lambda: pins.test_distill_gradient_matches_finite_differences(o, 0.7, 1)
    yield lambda: pins.test_distill_loss_matches_definition(o, 0.7, 1, 0)
    yield lambda: pins.test_distill_loss_matches_definition(o, 1.0, 2, 11)
    yield lambda: pins.test_distill_zero_when_target_equals_prediction(o)
    yield lambda: pins.test_distill_invariances_and_positivity(o)
    yield lambda: pins.test_tile_search_brute_force(o)
    yield lambda: pins.test_e4m3_format_facts(o)
    yield lambda: pins.test_e4m3_round_trip_midpoints_and_saturation(o)
    yield lambda: pins.test_e4m3_quantize_per_head(o)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name):
    old, new = MUTANTS[name]
    src = open(oracle_pkg._SRC).read()
    assert src.count(old) == 1, f"mutation site not unique: {old!r}"
    with tempfile.TemporaryDirectory() as tmp:
        path = os.path.join(tmp, "mutant.c")
        with open(path, "w") as f:
            f.write(src.replace(old, new))
        lib = oracle_pkg.load(oracle_pkg.build(path, os.path.join(tmp, "libmutant.so")))
        mutant = oracle_pkg.Oracle(lib)
        caught = False
        for pin in pin_suite(mutant):
            try:
                pin()
            except AssertionError:
                caught = True
                break
            except (ValueError, FloatingPointError, IndexError):
                caught = True
                break
        assert caught, f"no pin catches the mutant: {name}"


def test_unmutated_copy_passes_every_pin():
    src = open(oracle_pkg._SRC).read()
    with tempfile.TemporaryDirectory() as tmp:
        path = os.path.join(tmp, "copy.c")
        with open(path, "w") as f:
            f.write(src)
        lib = oracle_pkg.load(oracle_pkg.build(path, os.path.join(tmp, "libcopy.so")))
        o = oracle_pkg.Oracle(lib)
        for pin in pin_suite(o):
            pin()
