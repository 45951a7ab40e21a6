"""The oracle's pins must catch plausible mistakes.  Each case plants one
mistake in a temporary copy of the oracle's C source (on the CPU), builds it,
and runs the pin suite against it; the suite has to fail."""
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "moe_oracle.c")

MUTATIONS = {
    "weights_from_biased_scores": ("den += s[ord[j].i];", "den += m[ord[j].i];"),
    "bias_dropped_from_selection": ("m[i] = s[i] + (bias ? (double)bias[i] : 0.0);",
                                    "m[i] = s[i];"),
    "group_score_is_max": ("gs[g] = tmp[0] + tmp[1];", "gs[g] = tmp[0];"),
    "mask_value_swapped": ("m[i] = (mask_mode == 0) ? -INFINITY : 0.0;",
                           "m[i] = (mask_mode == 1) ? -INFINITY : 0.0;"),
    "ties_to_highest_index": ("return (a->i > b->i) - (a->i < b->i);",
                              "return (a->i < b->i) - (a->i > b->i);"),
    "no_renormalisation": ("w[j] = route_scale * (s[ord[j].i] / den);",
                           "w[j] = route_scale * s[ord[j].i];"),
    "unstable_dispatch": ("return (a->slot > b->slot) - (a->slot < b->slot);",
                          "return (a->slot < b->slot) - (a->slot > b->slot);"),
    "perm_inverse_swapped": ("inv[perm[i]] = (int32_t)i;", "inv[i] = perm[i];"),
    "routed_not_rounded": ("double routed = dtype == 1 ? mo_round_bf16(acc) : acc;",
                           "double routed = acc;"),
    "bf16_round_half_up": ("double r = nearbyint(ldexp(fabs(v), -q));",
                           "double r = floor(ldexp(fabs(v), -q) + 0.5);"),
    "logit_sign_flip": ("s[i] = 1.0 / (1.0 + exp(-acc));", "s[i] = 1.0 / (1.0 + exp(acc));"),
    "softmax_renormalised": ("w[j] = route_scale * s[ord[j].i];  /* softmax: not renormalised */",
                             "w[j] = route_scale * (s[ord[j].i] / den);"),
    "softmax_not_shifted_sum": ("sum += exp(L[i] - mx);", "sum += exp(L[i]);"),
    "group_max_is_pair_sum": ("gs[g] = tmp[0];\n            else", "gs[g] = tmp[0] + tmp[1];\n            else"),
    "epsilon_always_added": ("    if (var.eps)\n        den += 1e-20;", "    den += 1e-20;"),
    "one_group_too_few_kept": ("for (int r = topk_group; r < n_group; ++r) {",
                               "for (int r = topk_group - 1; r < n_group; ++r) {"),
    "margin_sign_flip": ("m_tok = ord[k - 1].v - ord[k].v;", "m_tok = ord[k].v - ord[k - 1].v;"),
    "offsets_start_at_first_count": ("offsets[0] = 0;", "offsets[0] = counts[0];"),
    "gather_token_is_slot_mod_k": ("long tok = perm[slot] / k;", "long tok = perm[slot] % k;"),
    "combine_weights_reversed": ("acc += (double)w[t * k + j] * mo_load(E, dtype, row * d + c);",
                                 "acc += (double)w[t * k + (k - 1 - j)] * "
                                 "mo_load(E, dtype, row * d + c);"),
    "combine_row_of_token_not_slot": ("long row = inv[t * k + j];", "long row = inv[t + j];"),
    "final_sum_not_rounded": ("                if (dtype == 1) y = mo_round_bf16(y);\n", ""),
    "expert_gemm_segment_off_by_one": ("while (offsets[e + 1] <= j) ++e;",
                                       "while (offsets[e + 1] < j) ++e;"),
    "expert_gemm_row_is_slot": ("const long tok = perm[j] / k;\n        for (int n = 0;",
                                "const long tok = perm[j] % T;\n        for (int n = 0;"),
    "ep_label_is_source": ("const int label = (int)(seg % E_loc);",
                           "const int label = (int)(seg / E_loc);"),
    "ep_recv_block_of_sender": ("const int32_t c = counts_all[(long)s * N_r + (long)r * E_loc + e];",
                                "const int32_t c = counts_all[(long)r * N_r + (long)s * E_loc + e];"),
    "ep_send_block_of_receiver": ("send += counts_all[(long)r * N_r + (long)s * E_loc + e];",
                                  "send += counts_all[(long)s * N_r + (long)r * E_loc + e];"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_mutation(name, tmp_path):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor not found once: {old}"
    mut = tmp_path / "moe_oracle_mut.c"
    mut.write_text(src.replace(old, new))
    lib = tmp_path / "liboracle_mut.so"
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                           "-o", str(lib), str(mut), "-lm"])
    env = dict(os.environ, MO_ORACLE_LIB=str(lib))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    # exit status 1: a pin failed (not a crash, a usage error or no tests)
    assert r.returncode == 1, (f"pins did not catch '{name}' (status {r.returncode}):\n"
                               f"{r.stdout[-2000:]}")
