"""Plant plausible mistakes in copies of the oracle source (on the CPU) and check that the pins catch each.

Every mutant is a textual edit of oracle/fa_oracle.c compiled into a temporary directory: a dropped term, a
wrong sign, a wrong index or operand, an off-by-one mask. The real oracle must pass every pin; each mutant
must fail at least one.
"""
import os

import pytest

import oracle_pins

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "fa_oracle.c")

MUTANTS = {
    "drop_scale": ("s[j] = scale * acc;", "s[j] = acc;"),
    "causal_off_by_one": ("if (m->causal && j > c) return 0;", "if (m->causal && j >= c) return 0;"),
    "causal_top_left": ("int64_t c = i + (m->Sk - m->Sq);", "int64_t c = i;"),
    "window_left_off_by_one": ("if (m->left >= 0 && j < c - m->left) return 0;",
                               "if (m->left >= 0 && j <= c - m->left) return 0;"),
    "window_right_ignored": ("if (m->right >= 0 && j > c + m->right) return 0;", ""),
    "gqa_wrong_kv_head": ("const double *kh = k + (h / group) * Sk * D;\n            const double *vh = v + (h / group) * Sk * D;",
                          "const double *kh = k + (h % n_kv_heads) * Sk * D;\n            const double *vh = v + (h % n_kv_heads) * Sk * D;"),
    "gqa_dk_not_summed": ("dkh[j * D + d] += scale * gk;", "dkh[j * D + d] = scale * gk;"),
    "lse_drops_max": ("double lse = m + log(sum);", "double lse = log(sum);"),
    "output_uses_k": ("o[d] += pz * vh[j * D + d];", "o[d] += pz * kh[j * D + d];"),
    "dp_uses_k": ("acc += doh[i * D + d] * vh[j * D + d];", "acc += doh[i * D + d] * kh[j * D + d];"),
    "ds_sign": ("dSi[j] = Pi[j] * (dP[j] - Di);", "dSi[j] = Pi[j] * (dP[j] + Di);"),
    "drop_Di": ("Di += Pi[j] * dP[j];", "Di += 0.0 * dP[j];"),
    "dq_no_scale": ("for (int64_t d = 0; d < D; ++d) dqi[d] *= scale;", ""),
    "dq_uses_v": ("dqi[d] += dSi[j] * kh[j * D + d];", "dqi[d] += dSi[j] * vh[j * D + d];"),
    "dk_uses_dout": ("gk += dS[r * Sk + j] * qh[i * D + d];", "gk += dS[r * Sk + j] * doh[i * D + d];"),
    "dv_uses_dS": ("gv += G[r * Sk + j] * doh[i * D + d];", "gv += dS[r * Sk + j] * doh[i * D + d];"),
    "dk_no_scale": ("dkh[j * D + d] += scale * gk;", "dkh[j * D + d] += gk;"),
    "philox_no_key_bump": ("k0 += PHILOX_W0;", ""),
    "philox_swapped_products": ("uint32_t n0 = (uint32_t)(p1 >> 32) ^ c1 ^ k0;", "uint32_t n0 = (uint32_t)(p0 >> 32) ^ c1 ^ k0;"),
    "dropout_word_byte_swapped": ("uint32_t byte = (w[i & 3] >> (8 * (j & 3))) & 0xffu;",
                                  "uint32_t byte = (w[j & 3] >> (8 * (i & 3))) & 0xffu;"),
    "dropout_threshold_flipped": ("return byte >= (uint32_t)dr->t ?", "return byte < (uint32_t)dr->t ?"),
    "dropout_no_rescale": ("? 1.0 / (1.0 - dr->t / 256.0) : 0.0;", "? 1.0 : 0.0;"),
    "dropout_counter_ignores_head": ("(uint32_t)(j >> 2), (uint32_t)bh, dr->offset};", "(uint32_t)(j >> 2), 0u, dr->offset};"),
    "dropout_dv_undropped": ("gv += G[r * Sk + j] * doh[i * D + d];", "gv += P[r * Sk + j] * doh[i * D + d];"),
    "dropout_dp_unmasked": ("dP[j] = z * acc;", "dP[j] = acc;"),
    "dropout_counter_rows_keys_swapped": ("(uint32_t)(i >> 2), (uint32_t)(j >> 2), (uint32_t)bh, dr->offset};",
                                          "(uint32_t)(j >> 2), (uint32_t)(i >> 2), (uint32_t)bh, dr->offset};"),
    "dropout_offset_ignored": ("(uint32_t)(j >> 2), (uint32_t)bh, dr->offset};", "(uint32_t)(j >> 2), (uint32_t)bh, 0u};"),
    "philox_key_words_swapped": ("uint32_t k0 = key[0], k1 = key[1];", "uint32_t k0 = key[1], k1 = key[0];"),
    "window_right_off_by_one": ("if (m->right >= 0 && j > c + m->right) return 0;",
                                "if (m->right >= 0 && j >= c + m->right) return 0;"),
    "max_over_masked_scores": ("if (visible(i, j, mk) && s[j] > m) m = s[j];", "if (s[j] > m) m = s[j];"),
    # the backward's rows are a listed subset: r indexes the list, i the absolute query row
    "bwd_scores_row_r": ("row_scores(qh + i * D, kh, Sk, D, scale, s);", "row_scores(qh + r * D, kh, Sk, D, scale, s);"),
    "bwd_mask_row_r": ("row_softmax(s, i, &mk, Pi);", "row_softmax(s, r, &mk, Pi);"),
    "dp_dout_row_r": ("for (int64_t d = 0; d < D; ++d) acc += doh[i * D + d] * vh[j * D + d];",
                      "for (int64_t d = 0; d < D; ++d) acc += doh[r * D + d] * vh[j * D + d];"),
    "dk_q_row_r": ("gk += dS[r * Sk + j] * qh[i * D + d];", "gk += dS[r * Sk + j] * qh[r * D + d];"),
    "dv_dout_row_r": ("gv += G[r * Sk + j] * doh[i * D + d];", "gv += G[r * Sk + j] * doh[r * D + d];"),
    "bwd_dk_wrong_kv_head": ("double *dkh = dk + (h / group) * Sk * D;", "double *dkh = dk + (h % n_kv_heads) * Sk * D;"),
    "bwd_dropout_head_number_ignored": ("double z = dropout_z(dr, head_number(head_index, h), i, j);",
                                        "double z = dropout_z(dr, h, i, j);"),
    "fwd_dropout_flat_row": ("double pz = p[j] * dropout_z(dr, head_number(head_index, h), i, j);",
                             "double pz = p[j] * dropout_z(dr, head_number(head_index, h), t, j);"),
    "dropout_threshold_truncated": ("int t = (int)floor(256.0 * p + 0.5);", "int t = (int)floor(256.0 * p);"),
    "dropout_threshold_scale_255": ("int t = (int)floor(256.0 * p + 0.5);", "int t = (int)floor(255.0 * p + 0.5);"),
    "dropout_threshold_accepts_256": ("return t <= 255 ? t : -1;", "return t <= 256 ? t : -1;"),
    "dk_transposed_index": ("gk += dS[r * Sk + j] * qh[i * D + d];", "gk += dS[r * Sk + j] * qh[j % Sq * D + d];"),
}


@pytest.fixture(scope="module")
def src_text():
    with open(SRC) as f:
        return f.read()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, src_text, tmp_path):
    import oracle
    from oracle import build as obuild

    old, new = MUTANTS[name]
    assert src_text.count(old) == 1, "mutation site not found exactly once: " + old
    mutated = src_text.replace(old, new)
    src = tmp_path / ("mutant_%s.c" % name)
    src.write_text(mutated)
    lib = obuild.build(str(src), str(tmp_path / ("libmutant_%s.so" % name)))
    orc = oracle.Oracle(lib)
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(orc)
        except (AssertionError, ValueError, FloatingPointError):
            caught.append(pin.__name__)
    assert caught, "no pin caught the mutant " + name
