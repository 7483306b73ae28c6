"""Plant plausible mistakes in a copy of the oracle and check the pins catch each.

The copy lives in a temporary directory and is compiled with the oracle's own
flags; the oracle source itself is never modified.
"""
import os
import subprocess

import pytest

import oracle
import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "fps_oracle.c")

MUTATIONS = {
    "drop_dt_term": ("    s = s + dt * dt;\n", ""),
    "reorder_sum": ("    float s = dx * dx + dy * dy;\n    s = s + dz * dz;\n    s = s + dt * dt;\n",
                    "    float s = dz * dz + dt * dt;\n    s = s + dy * dy;\n    s = s + dx * dx;\n"),
    "wrong_axis": ("    float dz = p[2] - c[2];\n", "    float dz = p[2] - c[1];\n"),
    "argmax_tie_highest": ("if (best < 0 || dist[i] > dist[best]) best = i;",
                           "if (best < 0 || dist[i] >= dist[best]) best = i;"),
    "argmax_includes_chosen": ("                if (chosen[i]) continue;\n", ""),
    "no_running_min": ("if (d < dist[i]) dist[i] = d;", "dist[i] = d;"),
    "centroid_not_offset": ("const float *pc = coords + 4 * (off + c);", "const float *pc = coords + 4 * c;"),
    "voronoi_tie_highest": ("if (lab < 0 || d < best) {", "if (lab < 0 || d <= best) {"),
    "knn_tie_highest": ("return (x->i > y->i) - (x->i < y->i);", "return (x->i < y->i) - (x->i > y->i);"),
    "lloyd_unweighted": ("W[j] += q;", "W[j] += 1.0;"),
    "lloyd_wrong_coord": ("S[4 * j + a] += q * (double)coords[4 * (off + i) + a];",
                          "S[4 * j + a] += q * (double)coords[4 * (off + i)];"),
    "pool_wrong_column": ("sum[(int64_t)j * F + f] += (double)feats[(off + i) * F + f];",
                          "sum[(int64_t)j * F + f] += (double)feats[(off + i) * F];"),
    "pool_bwd_no_count": ("g = (float)((double)grad_pooled[((int64_t)b * K + j) * F + f] / (double)c);",
                          "g = grad_pooled[((int64_t)b * K + j) * F + f];"),
    "pool_bwd_wrong_event": ("g = (float)((double)grad_pooled[((int64_t)b * K + j) * F + f] / (double)c);",
                             "g = (float)((double)grad_pooled[(int64_t)j * F + f] / (double)c);"),
    "philox_no_key_bump": ("            k0 += 0x9E3779B9u;\n", ""),
    "philox_swapped_words": ("uint32_t n0 = hi1 ^ c1 ^ k0, n1 = lo1, n2 = hi0 ^ c3 ^ k1, n3 = lo0;",
                             "uint32_t n0 = hi0 ^ c1 ^ k0, n1 = lo0, n2 = hi1 ^ c3 ^ k1, n3 = lo1;"),
    "summary_unweighted_coords": ("for (int c = 0; c < 4; ++c) a[1 + c] += q * (double)coords[4 * i + c];",
                                  "for (int c = 0; c < 4; ++c) a[1 + c] += (double)coords[4 * i + c];"),
    "summary_charge_from_col1": ("double q = charge_col >= 0 ? (double)feats[i * F + charge_col] : 1.0;",
                                 "double q = charge_col >= 0 ? (double)feats[i * F + 1] : 1.0;"),
    "pack_drops_last_token": ("        for (int64_t j = 0; j < v; ++j) {\n            int64_t t = tok_offsets[b] + j;",
                              "        for (int64_t j = 0; j + 1 < v; ++j) {\n            int64_t t = tok_offsets[b] + j;"),
    "unpack_no_zero_pad": ("j < v ? src[(tok_offsets[b] + j) * D + d] : 0.0f;",
                           "j < v ? src[(tok_offsets[b] + j) * D + d] : src[0];"),
    "scale_wrong_axis": ("        ps[a] = w[a] * p[a];\n        cs[a] = w[a] * c[a];\n",
                         "        ps[a] = w[3 - a] * p[a];\n        cs[a] = w[3 - a] * c[a];\n"),
    "scale_point_only": ("        cs[a] = w[a] * c[a];\n", "        cs[a] = c[a];\n"),
    "knn_bwd_first_feature": ("acc[(int64_t)i * F + f] += (double)grad_pooled[r * F + f] / (double)counts[r];",
                              "acc[(int64_t)i * F + f] += (double)grad_pooled[r * F] / (double)counts[r];"),
}

PINS = [
    pins.pin_dist_golden, pins.pin_dist_error_bound, pins.pin_fps_fixtures, pins.pin_fps_bruteforce,
    pins.pin_fps_invariants, pins.pin_assign_bruteforce, pins.pin_knn_bruteforce,
    pins.pin_pool_bruteforce, pins.pin_lloyd_closed_form, pins.pin_pool_backward_adjoint, pins.pin_pack_tokens, pins.pin_token_summaries, pins.pin_random_starts,
    pins.pin_axis_scale,
]


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTATIONS[name]
    text = open(SRC).read()
    assert text.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    path = tmp_path / "mutant.c"
    path.write_text(text.replace(old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", *oracle.CFLAGS, str(path), "-o", str(lib), "-lm"])
    caught = []
    with oracle.use_library(str(lib)):
        for pin in PINS:
            try:
                pin()
            except (AssertionError, ValueError):
                caught.append(pin.__name__)
    assert caught, f"no pin catches mutation {name}"
